"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check each is caught by a pin.

This is the evidence that the pins constrain every part of the oracle: a dropped term, a wrong
sign, index or base, a transposed operand or a swapped nibble each makes some pin fail.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import attention as A
from oracle import layout as Lay
from oracle import nvfp4 as N4
import _pins


def _attend_no_scale(q, K, V, scale):
    return A.attend(q, K, V, 1.0)


def _attend_lse_drops_max(q, K, V, scale):
    O, L = A.attend(q, K, V, scale)
    z = scale * (np.asarray(q, float) @ np.asarray(K, float).T) if len(K) else None
    return O, (L - z.max(1)) if z is not None else L


def _attend_unnormalised(q, K, V, scale):
    O, L = A.attend(q, K, V, scale)
    z = scale * (np.asarray(q, float) @ np.asarray(K, float).T) if len(K) else None
    if z is None:
        return O, L
    w = np.exp(z - z.max(1, keepdims=True))
    return O * w.sum(1, keepdims=True), L


def _attend_log2(q, K, V, scale):
    O, L = A.attend(q, K, V, scale)
    return O, L / math.log(2)


def _combine_unnormalised(O_s, lse_s):
    O, L = A.combine(O_s, lse_s)
    M = np.max(lse_s, 0)
    den = np.exp(np.asarray(lse_s) - np.where(np.isfinite(M), M, 0)).sum(0)
    return O * np.where(np.isfinite(M), den, 1)[..., None], L


def _combine_plain_mean(O_s, lse_s):
    O, L = A.combine(O_s, lse_s)
    return np.mean(O_s, 0), L


def _combine_sign(O_s, lse_s):
    return A.combine(O_s, -np.asarray(lse_s))


def _decode_wrong_group(q, K, V, seq_lens, scale):
    saved = A._group_of
    A._group_of = lambda h, hq, hkv: h % hkv
    try:
        return A.decode(q, K, V, seq_lens, scale)
    finally:
        A._group_of = saved


def _decode_transposed_k(q, K, V, seq_lens, scale):
    # uses K's head-dim reversed: a transposed/permuted operand
    return A.decode(q, np.asarray(K)[..., ::-1], V, seq_lens, scale)


def _rr_swap(t, P, block=16):
    j, r = divmod(int(t), block)
    return j // P if P > 1 else 0, (j % P) * block + r


def _rr_drop_offset(t, P, block=16):
    j, r = divmod(int(t), block)
    return j % P, (j // P) * block


def _rr_off_by_one(t, P, block=16):
    j, r = divmod(int(t) + 1, block)
    return j % P, (j // P) * block + r


def _e2m1_bias(code):
    code = int(code) & 0xF
    e, m = (code >> 1) & 3, code & 1
    mag = 0.5 * m if e == 0 else math.ldexp(1 + 0.5 * m, e - 2)
    return -mag if code & 8 else mag


def _e4m3_bias(byte):
    v = N4.e4m3_value(byte)
    return v * 0.5


def _dequant_swapped_nibbles(codes, scales):
    c = np.asarray(codes, dtype=np.uint8)
    return N4.nvfp4_dequant(((c & 0xF) << 4) | (c >> 4), scales)


def _dequant_scale_per_8(codes, scales):
    # scale j applied to elements 8j .. 8j+7 (wrong block size), last scale reused past the end
    x = N4.nvfp4_dequant(codes, np.zeros_like(np.asarray(scales)) + 0x38)
    s = np.asarray([[N4.e4m3_value(b) for b in row] for row in np.asarray(scales)])
    idx = np.minimum(np.arange(x.shape[1]) // 8, s.shape[1] - 1)
    return x * s[:, idx]


def _caught(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    except (ValueError, IndexError):
        return True
    return False


ATTEND_MUTANTS = [_attend_no_scale, _attend_lse_drops_max, _attend_unnormalised, _attend_log2]


@pytest.mark.parametrize("mut", ATTEND_MUTANTS, ids=lambda f: f.__name__)
def test_attend_mutants_caught(mut):
    assert (_caught(_pins.pin_brute_force, mut) or _caught(_pins.pin_closed_forms, mut)
            or _caught(_pins.pin_invariances, mut)), mut.__name__


@pytest.mark.parametrize("mut", [_combine_unnormalised, _combine_plain_mean, _combine_sign],
                         ids=lambda f: f.__name__)
def test_combine_mutants_caught(mut):
    assert _caught(_pins.pin_combine_identity, A.attend, mut, Lay.shard_tokens)


@pytest.mark.parametrize("mut", [_decode_wrong_group, _decode_transposed_k], ids=lambda f: f.__name__)
def test_decode_mutants_caught(mut):
    assert _caught(_pins.pin_torch_sdpa, mut)


@pytest.mark.parametrize("mut", [_rr_swap, _rr_drop_offset, _rr_off_by_one], ids=lambda f: f.__name__)
def test_layout_mutants_caught(mut):
    def shard_tokens(S, P, layout, block=16, chunk=None):
        out = [[] for _ in range(P)]
        for t in range(S):
            s, _ = mut(t, P, block) if layout == "rr" else Lay.contig_place(t, chunk)
            out[s].append(t)
        return [np.asarray(x) for x in out]

    assert _caught(_pins.pin_layout, mut, Lay.contig_place, shard_tokens, Lay.shard_lens, Lay.page_slot)


@pytest.mark.parametrize("which", ["e2m1", "e4m3", "nibbles", "scale_block"])
def test_nvfp4_mutants_caught(which):
    e2, e4, dq = N4.e2m1_value, N4.e4m3_value, N4.nvfp4_dequant
    if which == "e2m1":
        e2 = _e2m1_bias
    elif which == "e4m3":
        e4 = _e4m3_bias
    elif which == "nibbles":
        dq = _dequant_swapped_nibbles
    else:
        dq = _dequant_scale_per_8
    assert _caught(_pins.pin_nvfp4, e2, e4, dq)


def _enc_ties_away(x):
    saved = N4._nearest_even

    def away(a, table):
        d = np.abs(np.asarray(a, float)[..., None] - table)
        dmin = d.min(-1, keepdims=True)
        idx = np.arange(table.shape[0])
        return np.where(d == dmin, idx, -1).max(-1)  # larger entry on a tie
    N4._nearest_even = away
    try:
        return N4.nvfp4_encode(x)
    finally:
        N4._nearest_even = saved


def _enc_truncate(x):
    saved = N4._nearest_even

    def floor_(a, table):
        a = np.asarray(a, float)
        return (a[..., None] >= table).sum(-1) - 1
    N4._nearest_even = floor_
    try:
        return N4.nvfp4_encode(x)
    finally:
        N4._nearest_even = saved


def _enc_signed_max(x):
    x = np.asarray(x, np.float32)
    c, s = N4.nvfp4_encode(x)
    xb = x.reshape(*x.shape[:-1], -1, 16)
    r = (np.maximum(xb.max(-1), 0) / np.float32(6)).astype(np.float32)
    return c, N4.e4m3_encode_satfinite(r)


def _enc_no_clamp(x):
    x = np.asarray(x, np.float32)
    c, s = N4.nvfp4_encode(x)
    big = np.abs(x.reshape(*x.shape[:-1], -1, 16)).max(-1) / 6 > 448
    return c, np.where(big, np.uint8(0x7F), s)  # overflow to NaN instead of 448


def _enc_negative_zero(x):
    x = np.asarray(x, np.float32)
    c, s = N4.nvfp4_encode(x)
    neg = (x < 0).reshape(*x.shape[:-1], -1, 2)
    lo = np.where(((c & 0xF) == 0) & neg[..., 0], c | 0x8, c)
    return np.where(((lo >> 4) == 0) & neg[..., 1], lo | 0x80, lo).astype(np.uint8), s


def _enc_swapped_nibbles(x):
    c, s = N4.nvfp4_encode(x)
    return ((c & 0xF) << 4 | (c >> 4)).astype(np.uint8), s


@pytest.mark.parametrize("mut", [_enc_ties_away, _enc_truncate, _enc_signed_max, _enc_no_clamp,
                                 _enc_negative_zero, _enc_swapped_nibbles],
                         ids=lambda f: f.__name__)
def test_nvfp4_encode_mutants_caught(mut):
    assert _caught(_pins.pin_nvfp4_encode, mut)


def test_real_oracle_passes_every_pin():
    _pins.pin_brute_force(oracle.attend)
    _pins.pin_closed_forms(oracle.attend)
    _pins.pin_invariances(oracle.attend)
    _pins.pin_torch_sdpa(oracle.decode)
    _pins.pin_combine_identity(oracle.attend, oracle.combine, oracle.shard_tokens)
    _pins.pin_nvfp4_encode(oracle.nvfp4_encode)
