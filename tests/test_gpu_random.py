"""Seeded random shapes for every kernel (head dims, group sizes, shard counts, both layouts, ragged
lengths down to one token), each checked element by element against the oracle through the fused
partial + combine call and the per-shard partials."""

import numpy as np
import pytest
import torch

import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu


def _gqa_cases(n, kv_dtype, seed):
    rng = np.random.default_rng(seed)
    base = wl.WORKLOADS["gqa_s128k" if kv_dtype == "bf16" else "gqa_nvfp4_s1m"]
    out = []
    for i in range(n):
        d = 128 if kv_dtype == "nvfp4" else int(rng.choice([64, 128]))
        hkv = int(rng.integers(1, 4))
        g = int(rng.choice([1, 2, 4, 8, 16]))
        B = int(rng.integers(1, 4))
        kvp = int(rng.integers(1, 9))
        layout = str(rng.choice(["rr", "contig"]))
        S = int(rng.integers(64, 6000))
        lens = [int(x) for x in rng.integers(1, S + 1, size=B)]
        lens[int(rng.integers(0, B))] = S
        w = base.with_(name=f"{kv_dtype}_{i}", B=B, Hq=g * hkv, Hkv=hkv, d=d, dv=d, S=S, kvp=kvp,
                       layout=layout, seed=9000 + 97 * i + (0 if kv_dtype == "bf16" else 5000))
        out.append((w, lens))
    return out


def _mla_cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        B = int(rng.integers(1, 3))
        kvp = int(rng.integers(1, 9))
        S = int(rng.integers(64, 3000))
        lens = [int(x) for x in rng.integers(1, S + 1, size=B)]
        lens[0] = S
        w = wl.WORKLOADS["mla_s1m"].with_(name=f"mla_{i}", B=B, S=S, kvp=kvp, seed=9500 + 31 * i)
        out.append((w, lens))
    return out


CASES = _gqa_cases(8, "bf16", 1) + _gqa_cases(6, "nvfp4", 2) + _mla_cases(4, 3)


@pytest.mark.parametrize("case", range(len(CASES)), ids=[c[0].name for c in CASES])
def test_random_shape_against_oracle(case):
    w, lens = CASES[case]
    hx = _gpu.hx()
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=2048)
    assert cache.err_bits() == 0
    q = wl.query(w, "cuda")
    o_part = torch.empty(w.kvp, w.B, w.Hq, w.dv, device="cuda")
    lse_part = torch.empty(w.kvp, w.B, w.Hq, device="cuda")
    out, lse = hx.partial_combine(cache, q, w.softmax_scale, o_part, lse_part,
                                  out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    o_part, lse_part = o_part.cpu().numpy(), lse_part.cpu().numpy()
    label = f"{w.name} B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} kvp={w.kvp} {w.layout} lens={lens}"
    for b in range(w.B):
        for h in range(w.Hkv):
            O, L, Os, Ls = _gpu.oracle_head_group(w, q, b, h, lens[b])
            hs = slice(h * w.G, (h + 1) * w.G)
            _gpu.assert_close_O(out[b, hs], O, f"{label} O b={b} h={h}")
            _gpu.assert_close_lse(lse[b, hs], L, f"{label} LSE b={b} h={h}")
            _gpu.assert_close_O(o_part[:, b, hs], Os, f"{label} O_partial b={b} h={h}")
            _gpu.assert_close_lse(lse_part[:, b, hs], Ls, f"{label} lse_partial b={b} h={h}")
