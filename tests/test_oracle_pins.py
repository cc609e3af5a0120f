"""The oracle against what the pages and the mathematics fix (CPU only)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import _pins


def test_brute_force():
    _pins.pin_brute_force(oracle.attend)


def test_closed_forms():
    _pins.pin_closed_forms(oracle.attend)


def test_invariances():
    _pins.pin_invariances(oracle.attend)


def test_torch_sdpa_gqa():
    _pins.pin_torch_sdpa(oracle.decode)


def test_combine_identity():
    _pins.pin_combine_identity(oracle.attend, oracle.combine, oracle.shard_tokens)


def test_layout():
    _pins.pin_layout(oracle.rr_place, oracle.contig_place, oracle.shard_tokens,
                     oracle.shard_lens, oracle.page_slot)


def test_nvfp4_tables():
    _pins.pin_nvfp4(oracle.e2m1_value, oracle.e4m3_value, oracle.nvfp4_dequant)


def test_partial_then_combine_equals_decode_gqa():
    """Batch-level: per-shard partials for the round-robin-16 layout combine to the unsharded
    decode, with GQA head mapping, on bf16 inputs drawn by the workload generator."""
    w = wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=8, Hkv=2, d=32, dv=32, S=300, kvp=3)
    q = wl.query(w)
    K = torch.stack([wl.kv_tokens(w, "k", b, 0, w.S) for b in range(w.B)])
    V = torch.stack([wl.kv_tokens(w, "v", b, 0, w.S) for b in range(w.B)])
    lens = [300, 171]
    sets = [oracle.shard_tokens(S, w.kvp, "rr", 16) for S in lens]
    O, L = oracle.decode(q, K, V, lens, w.softmax_scale)
    Os, Ls = oracle.partial(q, K, V, sets, w.softmax_scale)
    Oc, Lc = oracle.combine(Os, Ls)
    np.testing.assert_allclose(Oc, O, atol=1e-13)
    np.testing.assert_allclose(Lc, L, atol=1e-12)


def test_mla_decode_matches_sdpa():
    """MLA reading: one latent head of width 576 is K, its first 512 columns are V."""
    g = torch.Generator().manual_seed(7)
    B, H, S, dk, dv = 2, 16, 40, 576, 512
    q = torch.randn(B, H, dk, generator=g, dtype=torch.float64)
    C = torch.randn(B, S, 1, dk, generator=g, dtype=torch.float64)
    sc = 1 / 24.0
    O, L = oracle.decode(q, C, C[..., :dv], [S] * B, sc)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, :, None], C.transpose(1, 2).expand(B, H, S, dk),
        C[..., :dv].transpose(1, 2).expand(B, H, S, dv), scale=sc)[:, :, 0]
    np.testing.assert_allclose(O, ref.numpy(), atol=1e-12)


def test_roofline_byte_model():
    """The byte model reproduces the pages' KV-read roofline (1,024 us at TP=1, 128 us at TP=8)."""
    for row in _pins._golden_rows("roofline_fp4_kv_read.txt"):
        tp, heads, B, T, d, eb, bw, us = row
        t = wl.kv_read_bytes(int(B) * int(T), int(heads), int(d), float(eb)) / float(bw) * 1e6
        assert abs(t - float(us)) < 1e-9


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_workload_bytes_positive(name):
    w = wl.WORKLOADS[name]
    lens = wl.seq_lens(w)
    assert all(1 <= s <= w.S for s in lens)
    assert wl.step_bytes(w, lens) > wl.partial_bytes(w, lens) > 0


def test_nvfp4_encode():
    _pins.pin_nvfp4_encode(oracle.nvfp4_encode)
