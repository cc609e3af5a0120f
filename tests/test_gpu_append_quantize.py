"""helix_kv_append_quantize: bf16 K/V rows encoded to NVFP4 on the device, bit-exact against the
oracle's encoder, placed where the oracle's layout rule puts them, and attended correctly."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu

W = wl.WORKLOADS["gqa_nvfp4_s1m"].with_(B=3, Hq=32, Hkv=2, S=700, kvp=4)
LENS = [700, 333, 65]


def _rows(w, seed):
    """bf16 rows [B, S, Hkv, 128]: N(0,1) blocks scaled over many binades, plus blocks that hit the
    encoder's edge cases (every E2M1 tie at scale 1, saturation, the 448 clamp, a zero scale, a
    subnormal scale, E4M3 scale ties, all zeros)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(w.B, w.S, w.Hkv, 8, 16, generator=g)
    x = x * torch.exp2(torch.randint(-16, 12, (w.B, w.S, w.Hkv, 8, 1), generator=g).float())
    special = torch.tensor([
        [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.2, -0.3, -6, 0, 4.4, 0.1, -5.5, 2.9],
        [6.2] + [0] * 14 + [-1],
        [3000, -3000] + [0] * 14,
        [1e-4, -1e-4] + [0] * 14,
        [0.01, 0.005] + [0] * 14,
        [6.375] + [0] * 15,
        [7.125, 1.25] + [0] * 14,
        [0] * 16,
    ], dtype=torch.float32)
    pick = torch.rand(w.B, w.S, w.Hkv, 8, generator=g) < 0.15
    which = torch.randint(0, special.shape[0], (w.B, w.S, w.Hkv, 8), generator=g)
    x = torch.where(pick[..., None], special[which], x)
    return x.reshape(w.B, w.S, w.Hkv, 128).to(torch.bfloat16)


def _fill_quantized(cache, k, v, lens, chunk):
    hx = _gpu.hx()
    for t0 in range(0, max(lens), chunk):
        n = min(chunk, max(lens) - t0)
        nv = torch.tensor([min(max(L - t0, 0), n) for L in lens], dtype=torch.int32, device="cuda")
        hx.append_quantize(cache, k[:, t0:t0 + n].contiguous(), v[:, t0:t0 + n].contiguous(),
                           n_valid=nv)
    torch.cuda.synchronize()


def _check_pools(w, cache, kc, ks, vc, vs, lens):
    """Every token's K codes / scales (natural rows) and V codes / scales (token-pair layout with
    the documented chunk swizzle, block-major scales) where the oracle's placement rule puts it."""
    kp, ksp = cache["k_pool"].cpu().numpy(), cache["k_scale"].cpu().numpy()
    vp, vsp = cache["v_pool"].cpu().numpy(), cache["v_scale"].cpu().numpy()
    pt = cache.page_table.cpu().numpy()
    col = np.arange(w.d)
    for b in range(w.B):
        for t in range(lens[b]):
            s, l_ = oracle.rr_place(t, w.kvp, w.rr_block)
            pi, slot = oracle.page_slot(l_)
            page = int(pt[s, b, pi])
            assert np.array_equal(kp[page, :, slot], kc[b, t]), ("k codes", b, t)
            assert np.array_equal(ksp[page, :, slot], ks[b, t]), ("k scales", b, t)
            assert np.array_equal(vsp[page, :, :, slot], vs[b, t]), ("v scales", b, t)
            want = np.stack([vc[b, t] & 0xF, vc[b, t] >> 4], -1).reshape(w.Hkv, w.d)
            pair = slot // 2
            pos = 16 * ((col // 16) ^ (2 * (pair % 4))) + col % 16
            got = (vp[page, :, pair, :][:, pos] >> (4 * (slot % 2))) & 0xF
            assert np.array_equal(got, want), ("v codes", b, t)


def test_append_quantize_bit_exact_against_the_oracle_encoder():
    w, lens = W, LENS
    k, v = _rows(w, 101).cuda(), _rows(w, 202).cuda()
    cache = _gpu.make_cache(w)
    # a ragged bulk append, then single-token appends (the decode case)
    _fill_quantized(cache, k, v, [L - 2 for L in lens], chunk=256)
    hx = _gpu.hx()
    for j in range(2):
        idx = [L - 2 + j for L in lens]
        k1 = torch.stack([k[b, idx[b]] for b in range(w.B)])[:, None].contiguous()
        v1 = torch.stack([v[b, idx[b]] for b in range(w.B)])[:, None].contiguous()
        hx.append_quantize(cache, k1, v1)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    assert cache["seq_lens"].tolist() == lens
    kc, ks = oracle.nvfp4_encode(k.float().cpu())
    vc, vs = oracle.nvfp4_encode(v.float().cpu())
    _check_pools(w, cache, kc, ks, vc, vs, lens)


def test_append_quantize_then_attend():
    """A history encoded on the device is attended exactly as the oracle attends the decoded
    oracle encoding of the same bf16 rows."""
    w, lens = W, LENS
    k, v = _rows(w, 303).cuda(), _rows(w, 404).cuda()
    # values of the size the tolerance is stated for (|V| of order 1; weights rounded to f16
    # move O by up to 2^-11 of |V|)
    k, v = k.clamp(-6, 6), v.clamp(-4, 4)
    cache = _gpu.make_cache(w)
    _fill_quantized(cache, k, v, lens, chunk=200)
    hx = _gpu.hx()
    q = wl.query(w, "cuda")
    o_part, lse_part = hx.partial(cache, q, w.softmax_scale)
    out, lse = hx.combine(o_part, lse_part, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    K = oracle.nvfp4_dequant(*oracle.nvfp4_encode(k.float().cpu()))
    V = oracle.nvfp4_dequant(*oracle.nvfp4_encode(v.float().cpu()))
    O, L = oracle.decode(q, K, V, lens, w.softmax_scale)
    _gpu.assert_close_O(out.cpu().numpy(), O, "O")
    _gpu.assert_close_lse(lse.cpu().numpy(), L, "LSE")


def test_append_quantize_rejects_bf16_caches():
    w = wl.WORKLOADS["gqa_s128k"].with_(B=1, Hq=16, Hkv=1, S=64, kvp=2)
    cache = _gpu.make_cache(w)
    x = torch.zeros(1, 1, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_gpu.hx().HelixError):
        _gpu.hx().append_quantize(cache, x, x)
