"""Request-range partial/combine and the two-stream HOP-B analogue (batch-wise overlap of one request
group's combine with the next group's partial attention), through the C ABI, against the oracle."""

import numpy as np
import pytest
import torch

import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu

GQA = wl.WORKLOADS["gqa_s128k"].with_(B=5, S=3000, kvp=4)
GQA_LENS = [3000, 17, 1200, 2999, 64]
MLA = wl.WORKLOADS["mla_s1m"].with_(B=3, S=2500, kvp=4)
MLA_LENS = [2500, 900, 33]
# Consistency between two launches that split the same units differently (see the range test)
SPLIT_TOL_O = 1e-2
SPLIT_TOL_LSE = 1e-4


def _setup(w, lens):
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=4096)
    assert cache.err_bits() == 0
    return cache, wl.query(w, "cuda")


def _check_requests(w, cache, q, lens, out, lse, reqs, label):
    """out / lse: combined O and LSE (host arrays); checks the listed requests against the oracle."""
    for b in reqs:
        for h in range(w.Hkv):
            O, L, _, _ = _gpu.oracle_head_group(w, q, b, h, lens[b])
            rows = slice(h * w.G, (h + 1) * w.G)
            _gpu.assert_close_O(out[b, rows], O, f"{label} O b={b} kvh={h}")
            _gpu.assert_close_lse(lse[b, rows], L, f"{label} LSE b={b} kvh={h}")


@pytest.mark.parametrize("w,lens", [(GQA, GQA_LENS), (MLA, MLA_LENS)], ids=["gqa", "mla"])
def test_partial_range_touches_only_its_requests(w, lens):
    hx = _gpu.hx()
    cache, q = _setup(w, lens)
    P, B, Hq, dv = w.kvp, w.B, w.Hq, w.dv
    o_part = torch.full((P, B, Hq, dv), float("nan"), device="cuda")
    lse = torch.full((P, B, Hq), float("nan"), device="cuda")
    hx.partial_range(cache, q, w.softmax_scale, 1, 2 if B == 3 else 3, o_part, lse)
    torch.cuda.synchronize()
    b1 = 2 if B == 3 else 3
    inside = list(range(1, b1))
    outside = [b for b in range(B) if b not in inside]
    assert torch.isnan(o_part[:, outside]).all() and torch.isnan(lse[:, outside]).all()
    # the requests in range equal a full-batch call up to the split rounding; check the oracle
    o_full, lse_full = hx.partial(cache, q, w.softmax_scale)
    out, lse_o = hx.combine(o_part, lse, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _check_requests(w, cache, q, lens, out.cpu().numpy(), lse_o.cpu().numpy(), inside, "range")
    # Against the full-batch call: the kernels split units across CTAs differently, so the
    # reference maximum each segment rounds its weights against differs; with bf16 weights (2^-9
    # relative rounding) O may move by a few 1e-4, while the fp32 LSE sums agree to fp32 rounding.
    assert (o_part[:, inside] - o_full[:, inside]).abs().max().item() < SPLIT_TOL_O
    fin = torch.isfinite(lse_full[:, inside])
    assert torch.equal(fin, torch.isfinite(lse[:, inside]))
    assert (lse[:, inside][fin] - lse_full[:, inside][fin]).abs().max().item() < SPLIT_TOL_LSE


def test_combine_range_is_bit_identical_to_full_combine():
    hx = _gpu.hx()
    w, lens = GQA, GQA_LENS
    cache, q = _setup(w, lens)
    o_part, lse = hx.partial(cache, q, w.softmax_scale)
    full, full_lse = hx.combine(o_part, lse)
    out = torch.full_like(full, float("nan"))
    lse_out = torch.full_like(full_lse, float("nan"))
    hx.combine_range(o_part, lse, 2, 4, out, lse_out)
    torch.cuda.synchronize()
    assert torch.equal(out[2:4], full[2:4]) and torch.equal(lse_out[2:4], full_lse[2:4])
    assert torch.isnan(out[:2].float()).all() and torch.isnan(out[4:].float()).all()
    assert torch.isnan(lse_out[:2]).all() and torch.isnan(lse_out[4:]).all()


@pytest.mark.parametrize("w,lens,groups", [(GQA, GQA_LENS, 1), (GQA, GQA_LENS, 2),
                                           (GQA, GQA_LENS, 5), (GQA, GQA_LENS, 9),
                                           (MLA, MLA_LENS, 3)],
                         ids=["gqa-g1", "gqa-g2", "gqa-g5", "gqa-g9-clamped", "mla-g3"])
def test_overlapped_matches_oracle_and_repeats_bit_identically(w, lens, groups):
    hx = _gpu.hx()
    cache, q = _setup(w, lens)
    ov = hx.Overlap(groups)
    a = [t.clone() for t in hx.overlapped(cache, q, w.softmax_scale, ov, out_dtype=torch.float32)]
    b = hx.overlapped(cache, q, w.softmax_scale, ov, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    _check_requests(w, cache, q, lens, a[0].cpu().numpy(), a[1].cpu().numpy(), range(w.B),
                    f"overlapped g={groups}")
    # against the serial step: same math, rounding differs only where a unit is split differently
    o_part, lse = hx.partial(cache, q, w.softmax_scale)
    ser, ser_lse = hx.combine(o_part, lse, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (a[0] - ser).abs().max().item() < SPLIT_TOL_O
    assert (a[1] - ser_lse).abs().max().item() < SPLIT_TOL_LSE
    assert cache.err_bits() == 0


def test_overlapped_orders_against_later_work_on_stream_a():
    """Work issued on the caller's stream after the overlapped call sees the combined output (the
    call joins stream B back into stream A)."""
    hx = _gpu.hx()
    w, lens = GQA, GQA_LENS
    cache, q = _setup(w, lens)
    ov = hx.Overlap(3)
    out = torch.zeros(w.B, w.Hq, w.dv, dtype=torch.float32, device="cuda")
    snap = torch.empty_like(out)
    for _ in range(3):
        out.zero_()
        hx.overlapped(cache, q, w.softmax_scale, ov, out=out)
        snap.copy_(out)  # same stream as the call
    torch.cuda.synchronize()
    o_part, lse = hx.partial(cache, q, w.softmax_scale)
    ser, ser_lse = hx.combine(o_part, lse, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert (snap - ser).abs().max().item() < SPLIT_TOL_O
    assert np.isfinite(snap.cpu().numpy()).all()
    _check_requests(w, cache, q, lens, snap.cpu().numpy(), ser_lse.cpu().numpy(), range(w.B),
                    "after overlapped")


@pytest.mark.parametrize("w,lens,groups", [(GQA, GQA_LENS, 2), (GQA, GQA_LENS, 5), (MLA, MLA_LENS, 2)],
                         ids=["gqa-g2", "gqa-g5", "mla-g2"])
def test_decode_overlapped_equals_the_serial_step(w, lens, groups):
    """HOP-B with the append overlapped too: per request group the new token is appended on the
    second stream while the previous group's partial runs. Same cache contents, lengths and (up to
    the split rounding) outputs as the serial decode step."""
    hx = _gpu.hx()
    ca, q = _setup(w, [L - 1 for L in lens])
    cb, _ = _setup(w, [L - 1 for L in lens])
    rows = _gpu.new_rows(w, 0, w.S)
    last = {k: torch.stack([v[b, lens[b] - 1] for b in range(w.B)])[:, None].contiguous()
            for k, v in rows.items()}
    out_a, lse_a = hx.decode_step(ca, q, last["k_new"], last.get("v_new"), w.softmax_scale,
                                  out=torch.empty(w.B, w.Hq, w.dv, device="cuda"))
    ov = hx.Overlap(groups)
    out_b, lse_b = hx.decode_overlapped(cb, q, w.softmax_scale, ov, last["k_new"], last.get("v_new"),
                                        out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ca["seq_lens"].tolist() == lens and cb["seq_lens"].tolist() == lens
    assert torch.equal(ca["shard_lens"], cb["shard_lens"])
    assert torch.equal(ca["k_pool"], cb["k_pool"])
    if w.kind != "mla":
        assert torch.equal(ca["v_pool"], cb["v_pool"])
    assert (out_a - out_b).abs().max().item() < SPLIT_TOL_O
    assert (lse_a - lse_b).abs().max().item() < SPLIT_TOL_LSE
    _check_requests(w, cb, q, lens, out_b.cpu().numpy(), lse_b.cpu().numpy(), range(w.B),
                    f"decode overlapped g={groups}")
    assert ca.err_bits() == 0 and cb.err_bits() == 0
