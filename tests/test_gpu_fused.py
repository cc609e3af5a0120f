"""helix_attn_partial_combine: the partial attention and the LSE combine in one launch (GQA), checked
bit-for-bit against the two separate calls and against the oracle."""

import numpy as np
import pytest
import torch

import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu

BF = wl.WORKLOADS["gqa_s128k"]
NV = wl.WORKLOADS["gqa_nvfp4_s1m"]
MLA = wl.WORKLOADS["mla_s1m"]

CASES = {
    # ragged lengths, one request shorter than a page, empty shards
    "bf16_ragged": (BF.with_(B=3, Hq=48, Hkv=3, S=3000), [3000, 40, 777]),
    # units split across CTAs (merged by tickets) before the group merge
    "bf16_split": (BF.with_(B=2, Hq=32, Hkv=2, S=90000, kvp=4), [90000, 61234]),
    # one shard: the short-context case, where the merge is the identity
    "bf16_kvp1": (BF.with_(B=2, Hq=16, Hkv=2, S=3500, kvp=1), [3500, 1000]),
    # head dim 64, contiguous layout (the tiny workload's shape)
    "bf16_tiny": (wl.WORKLOADS["tiny_gqa"], [4096]),
    "nvfp4_ragged": (NV.with_(B=3, Hq=32, Hkv=2, S=5000), [5000, 1, 2222]),
    "nvfp4_split": (NV.with_(B=1, Hq=16, Hkv=2, S=70000, kvp=2), [70000]),
    # MLA: the call falls back to two launches
    "mla": (MLA.with_(B=2, S=3000, kvp=4), [3000, 1500]),
}


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_fused_equals_separate_calls_and_oracle(name, out_dtype):
    w, lens = CASES[name]
    hx = _gpu.hx()
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=8192)
    q = wl.query(w, "cuda")
    ws = cache.workspace(w.Hq)
    o_sep, l_sep = hx.partial(cache, q, w.softmax_scale, workspace=ws)
    out_sep, lse_sep = hx.combine(o_sep, l_sep, out_dtype=out_dtype)
    results = []
    for _ in range(2):  # twice: the group tickets must be back at zero after a launch
        o_part = torch.full_like(o_sep, float("nan"))
        lse = torch.full_like(l_sep, float("nan"))
        out, lse_out = hx.partial_combine(cache, q, w.softmax_scale, o_part, lse,
                                          out_dtype=out_dtype, workspace=ws)
        torch.cuda.synchronize()
        results.append((o_part, lse, out, lse_out))
        assert torch.equal(o_part, o_sep) and torch.equal(lse, l_sep)
        assert torch.equal(out, out_sep) and torch.equal(lse_out, lse_sep)
    assert cache.err_bits() == 0
    # against the oracle, every request and head group
    out = results[0][2].float().cpu().numpy()
    lse_o = results[0][3].cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            O, L, _, _ = _gpu.oracle_head_group(w, q, b, h, lens[b])
            hs = slice(h * w.G, (h + 1) * w.G)
            _gpu.assert_close_O(out[b, hs], O, f"{name} O b={b} h={h}")
            _gpu.assert_close_lse(lse_o[b, hs], L, f"{name} LSE b={b} h={h}")


def test_fused_group_tickets_reset_and_workspace_reusable():
    w, lens = CASES["bf16_split"]
    hx = _gpu.hx()
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=8192)
    q = wl.query(w, "cuda")
    ws = cache.workspace(w.Hq)
    a = hx.partial_combine(cache, q, w.softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    # the ticket regions (unit tickets, then group tickets) are back to zero
    n_units = w.B * w.Hkv * w.kvp
    unit_bytes = -(-n_units * 4 // 256) * 256
    grp_bytes = -(-w.B * w.Hkv * 4 // 256) * 256
    assert int(ws[: unit_bytes + grp_bytes].view(torch.int32).abs().sum()) == 0
    b = hx.partial_combine(cache, q, w.softmax_scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
