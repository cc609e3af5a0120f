"""Input generators: determinism, block-independence and the NVFP4 encoder's contract."""

import numpy as np
import torch

import oracle
import workloads as wl


def test_kv_range_is_block_invariant():
    w = wl.WORKLOADS["gqa_s128k"].with_(d=16)
    full = wl.kv_range_f32(w, "k", 1, 3, 0, 3 * wl.GEN_BLOCK)
    part = wl.kv_range_f32(w, "k", 1, 3, wl.GEN_BLOCK - 5, 2 * wl.GEN_BLOCK + 7)
    assert torch.equal(part, full[wl.GEN_BLOCK - 5: 2 * wl.GEN_BLOCK + 7])
    again = wl.kv_range_f32(w, "k", 1, 3, 0, 10)
    assert torch.equal(again, full[:10])
    other = wl.kv_range_f32(w, "v", 1, 3, 0, 10)
    assert not torch.equal(other, full[:10])


def test_seq_lens_variable_range():
    w = wl.WORKLOADS["gqa_s1m_var"]
    lens = wl.seq_lens(w)
    assert lens == wl.seq_lens(w)
    assert all((1 << 19) <= s <= (1 << 20) for s in lens) and len(set(lens)) > 1


def test_page_table_is_a_permutation():
    w = wl.WORKLOADS["gqa_s128k"]
    pt, n = wl.page_table(w)
    assert pt.shape == (8, 8, 256)
    assert torch.equal(torch.sort(pt.flatten()).values, torch.arange(n, dtype=torch.int32))


def test_nvfp4_encoder_contract():
    """decode(encode(x)) lies on the scaled E2M1 grid, within half a grid step of x, and the block
    scale is absmax/6 rounded to E4M3."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(64, 128, generator=g) * torch.rand(64, 1, generator=g) * 10
    x[3, 16:32] = 0.0  # a zero block
    codes, scales = wl.nvfp4_encode(x)
    assert codes.dtype == torch.uint8 and codes.shape == (64, 64) and scales.shape == (64, 8)
    xh = oracle.nvfp4_dequant(codes.numpy(), scales.numpy())
    sc = np.repeat(np.array([[oracle.e4m3_value(b) for b in row] for row in scales.numpy()]), 16, 1)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    xb = x.numpy().astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(sc > 0, np.abs(xh) / np.where(sc > 0, sc, 1), 0)
    assert np.all(np.isin(ratio, grid))
    # nearest grid point: error at most half the local spacing (1 above 4.0, 0.5 in [2,4], 0.25 below)
    step = np.where(np.abs(xh) >= 4 * sc, 1.0, np.where(np.abs(xh) >= 2 * sc, 0.5, 0.25)) * sc
    assert np.all(np.abs(xh - xb) <= step + 1e-12)
    assert np.all(xh[3, 16:32] == 0) and scales[3, 1] == 0
    amax = np.abs(xb.reshape(64, 8, 16)).max(-1)
    want = torch.from_numpy(amax / 6).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(scales.numpy(), want)


def test_query_is_bf16_of_normal():
    w = wl.WORKLOADS["tiny_gqa"]
    q = wl.query(w)
    assert q.dtype == torch.bfloat16 and q.shape == (1, 8, 64)
    assert torch.equal(q, wl.query(w))
