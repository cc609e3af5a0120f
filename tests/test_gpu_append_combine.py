"""helix_kv_append placement (bit-exact against the oracle's layout rule) and helix_attn_combine
against the oracle's combine, on the GPU."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu


def _expected_pool(w, cache, rows_by_b, lens, stream="k"):
    """Where the oracle's placement rule puts every token, read back from the pool."""
    pool = cache[f"{stream}_pool"].cpu()
    pt = cache.page_table.cpu()
    for b in range(w.B):
        for t in range(lens[b]):
            s, l_ = oracle.contig_place(t, w.contig_chunk) if w.layout == "contig" else \
                oracle.rr_place(t, w.kvp, w.rr_block)
            pi, slot = oracle.page_slot(l_, w.page_tokens)
            page = int(pt[s, b, pi])
            got = pool[page, slot] if w.kind == "mla" else pool[page, :, slot]
            want = rows_by_b[b][t]
            assert torch.equal(got.view(torch.uint8), want.view(torch.uint8)), (b, t, s, l_)


@pytest.mark.parametrize("cfg", ["rr_bf16", "contig_bf16", "nvfp4", "mla"])
def test_append_bit_exact(cfg):
    if cfg == "rr_bf16":
        w = wl.WORKLOADS["gqa_s128k"].with_(B=3, Hq=16, Hkv=2, S=700, kvp=3)
    elif cfg == "contig_bf16":
        w = wl.WORKLOADS["tiny_gqa"].with_(B=2, S=500)
    elif cfg == "nvfp4":
        w = wl.WORKLOADS["gqa_nvfp4_s1m"].with_(B=2, Hq=16, Hkv=2, S=300, kvp=4)
    else:
        w = wl.WORKLOADS["mla_s1m"].with_(B=2, S=333, kvp=4)
    lens = [w.S - 17 * b for b in range(w.B)]
    cache = _gpu.make_cache(w)
    # a bulk append (ragged), then single-token appends
    _gpu.fill(cache, w, [L - 3 for L in lens], chunk=128)
    allrows = _gpu.new_rows(w, 0, w.S)
    hx = _gpu.hx()
    for j in range(3):
        one = {}
        for key, val in allrows.items():
            one[key] = torch.stack([val[b, lens[b] - 3 + j] for b in range(w.B)])[:, None].contiguous()
        hx.append(cache, **one)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    assert cache["seq_lens"].tolist() == lens
    want_shards = [oracle.shard_lens(L, w.kvp, w.layout, w.rr_block, w.contig_chunk) for L in lens]
    assert cache["shard_lens"].t().tolist() == want_shards
    if w.kind == "mla":
        _expected_pool(w, cache, [allrows["k_new"][b].cpu() for b in range(w.B)], lens, "k")
    elif w.kv_dtype == "bf16":
        for st, key in (("k", "k_new"), ("v", "v_new")):
            _expected_pool(w, cache, [allrows[key][b].cpu() for b in range(w.B)], lens, st)
    else:
        # K codes and K scales: natural rows. V codes: byte [slot // 2][c] holds element c of the
        # token in nibble slot % 2. V scales: [block][slot].
        _expected_pool(w, cache, [allrows["k_new"][b].cpu() for b in range(w.B)], lens, "k")
        ks, vp, vs = cache["k_scale"].cpu(), cache["v_pool"].cpu(), cache["v_scale"].cpu()
        pt = cache.page_table.cpu()
        for b in range(w.B):
            for t in range(lens[b]):
                s, l_ = oracle.rr_place(t, w.kvp, w.rr_block)
                pi, slot = oracle.page_slot(l_)
                page = int(pt[s, b, pi])
                assert torch.equal(ks[page, :, slot], allrows["k_scale"][b, t].cpu())
                assert torch.equal(vs[page, :, :, slot], allrows["v_scale"][b, t].cpu())
                src = allrows["v_new"][b, t].cpu().to(torch.int32)  # [H, d/2] natural packing
                codes = torch.stack([src & 0xF, src >> 4], -1).reshape(w.Hkv, w.d)
                pair = slot // 2
                col = torch.arange(w.d)
                pos = 16 * ((col // 16) ^ (2 * (pair % 4))) + col % 16  # documented swizzle
                got = (vp[page, :, pair, :][:, pos].to(torch.int32) >> (4 * (slot % 2))) & 0xF
                assert torch.equal(got, codes), (b, t)


def test_append_capacity_and_bad_page_errors():
    w = wl.WORKLOADS["gqa_s128k"].with_(B=1, Hq=16, Hkv=1, S=256, kvp=2)
    cache = _gpu.make_cache(w)  # room for 128 tokens per shard
    hx = _gpu.hx()
    rows = _gpu.new_rows(w, 0, 256)
    hx.append(cache, **rows)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    one = {k: v[:, :1].contiguous() for k, v in rows.items()}
    hx.append(cache, **one)  # token 256 -> shard 0, local 128: past the page table
    torch.cuda.synchronize()
    assert cache.err_bits() & hx.DEVERR_CAPACITY
    cache.clear_errors()
    cache.page_table[1, 0, 0] = -5
    w2 = w.with_(S=40)
    c2 = _gpu.make_cache(w2)
    c2.page_table[1, 0, 0] = -5
    hx.append(c2, **_gpu.new_rows(w2, 0, 40))
    torch.cuda.synchronize()
    assert c2.err_bits() & hx.DEVERR_PAGE_ID


@pytest.mark.parametrize("P,dv,out_dtype", [(8, 128, torch.float32), (3, 64, torch.bfloat16),
                                            (1, 512, torch.float32), (16, 4, torch.float32)])
def test_combine_matches_oracle(P, dv, out_dtype):
    g = torch.Generator().manual_seed(P * 1000 + dv)
    B, H = 3, 5
    Os = torch.randn(P, B, H, dv, generator=g)
    Ls = torch.randn(P, B, H, generator=g) * 3 + 10
    if P > 1:
        Ls[0, 0, 0] = -float("inf")  # an empty shard
        Ls[:, 1, 2] = -float("inf")  # every shard empty
    hx = _gpu.hx()
    out, lse = hx.combine(Os.cuda(), Ls.cuda(), out_dtype=out_dtype)
    torch.cuda.synchronize()
    O, L = oracle.combine(Os.numpy(), Ls.numpy())
    got = out.float().cpu().numpy()
    tol = 1e-5 if out_dtype == torch.float32 else 2 ** -8 * np.abs(O).max()
    assert np.abs(got - O).max() <= tol
    both = np.isneginf(L) & np.isneginf(lse.cpu().numpy())
    with np.errstate(invalid="ignore"):
        assert np.all(np.where(both, 0, np.abs(lse.cpu().numpy() - L)) <= 1e-5)
    if P > 1:
        assert np.all(got[1, 2] == 0) and np.isneginf(lse[1, 2].item())
