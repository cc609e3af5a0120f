"""MLA (absorbed, one 576-wide latent head, values = its first 512 columns) decode attention on the
GPU against the fp64 oracle. Same tolerances as the GQA tests."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu

MLA = wl.WORKLOADS["mla_s1m"]


def _run(cache, w, q):
    hx = _gpu.hx()
    o_part, lse_part = hx.partial(cache, q, w.softmax_scale)
    out, lse = hx.combine(o_part, lse_part, out_dtype=torch.float32)
    torch.cuda.synchronize()
    return o_part.cpu().numpy(), lse_part.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def _check(w, q, lens, res, label, heads=None):
    o_part, lse_part, out, lse = res
    heads = list(range(w.Hq)) if heads is None else heads
    for b in range(w.B):
        C = oracle.attention._f64(wl.kv_range_bf16(w, "c", b, 0, 0, lens[b], "cuda"))
        qb = oracle.attention._f64(q[b, heads])
        O, L = oracle.attend(qb, C, C[:, : w.dv], w.softmax_scale)
        _gpu.assert_close_O(out[b, heads], O, f"{label} O b={b}")
        _gpu.assert_close_lse(lse[b, heads], L, f"{label} LSE b={b}")
        for s, idx in enumerate(_gpu.shard_sets(w, lens[b])):
            Os, Ls = oracle.attend(qb, C[idx], C[idx][:, : w.dv], w.softmax_scale)
            _gpu.assert_close_O(o_part[s, b, heads], Os, f"{label} O_partial b={b} s={s}")
            _gpu.assert_close_lse(lse_part[s, b, heads], Ls, f"{label} lse_partial b={b} s={s}")


CASES = {
    # several 64-token tiles and a partial tile per shard
    "small": (MLA.with_(B=1, S=700, kvp=2), [700]),
    # one token, a partial page, empty shards (8 shards, 1 token)
    "ragged_empty": (MLA.with_(B=3, S=1000, kvp=8), [1000, 1, 77]),
    # long enough that every unit is split across several clusters and merged by tickets
    "split_units": (MLA.with_(B=2, S=40000, kvp=2), [40000, 25000]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_mla_small(name):
    w, lens = CASES[name]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=4096)
    assert cache.err_bits() == 0
    q = wl.query(w, "cuda")
    _check(w, q, lens, _run(cache, w, q), name)
    assert cache.err_bits() == 0


def test_mla_sharp_query_and_repeat():
    """A sharp query (q x 8) makes the softmax nearly one-hot (|O| of order |V|) and exercises the
    lazy rescale; two calls must be bit-identical."""
    w = MLA.with_(B=2, S=6000, kvp=4)
    lens = [6000, 3333]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=4096)
    q = wl.query(w, "cuda", scale_by=8.0)
    a = _run(cache, w, q)
    b = _run(cache, w, q)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    _check(w, q, lens, a, "sharp")
    assert np.abs(a[2]).max() > 0.3


def test_mla_decode_step():
    w = MLA.with_(B=2, S=3000, kvp=8)
    lens0 = [2990, 1500]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens0, chunk=1024)
    rows = _gpu.new_rows(w, 0, w.S)
    hx = _gpu.hx()
    q = wl.query(w, "cuda")
    for step in range(3):
        k1 = torch.stack([rows["k_new"][b, lens0[b] + step] for b in range(w.B)])[:, None]
        out, lse = hx.decode_step(cache, q, k1.contiguous(), None, w.softmax_scale)
        torch.cuda.synchronize()
        lens = [L + step + 1 for L in lens0]
        C = rows["k_new"].cpu()
        O, L = oracle.decode(q, C[:, :, None], C[:, :, None, : w.dv], lens, w.softmax_scale)
        _gpu.assert_close_O(out.float().cpu().numpy(), O, f"step {step}")
        _gpu.assert_close_lse(lse.cpu().numpy(), L, f"step {step}")


def test_mla_full_1m_sampled():
    """The full 1M-token MLA workload in the benchmark's launch configuration, eight sampled heads
    of two requests (the oracle holds a 1M x 576 fp64 latent per request)."""
    w = MLA
    lens = wl.seq_lens(w)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens)
    assert cache.err_bits() == 0
    q = wl.query(w, "cuda")
    hx = _gpu.hx()
    o_part, lse_part = hx.partial(cache, q, w.softmax_scale)
    out, lse = hx.combine(o_part, lse_part)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    heads = [0, 37, 64, 127]
    for b in (0, 7):
        C = oracle.attention._f64(wl.kv_range_bf16(w, "c", b, 0, 0, lens[b], "cuda"))
        qb = oracle.attention._f64(q[b, heads])
        O, L = oracle.attend(qb, C, C[:, : w.dv], w.softmax_scale)
        _gpu.assert_close_O(out[b, heads].float().cpu().numpy(), O, f"O b={b}")
        _gpu.assert_close_lse(lse[b, heads].cpu().numpy(), L, f"LSE b={b}")
        del C
    del cache
    torch.cuda.empty_cache()


def test_mla_bad_page_id_sets_error_and_skips():
    """A page id outside the pool sets the device error bit, and that page's 64 tokens are left out
    of its shard (masked scores, zeroed values); the rest of the shard is attended exactly."""
    w = MLA.with_(B=1, S=640, kvp=2)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, [640])
    cache.page_table[1, 0, 2] = 10 ** 6  # beyond the pool: local tokens 128..191 of shard 1
    cache.clear_errors()
    q = wl.query(w, "cuda")
    o_part, lse_part, _, _ = _run(cache, w, q)
    assert cache.err_bits() & _gpu.hx().DEVERR_PAGE_ID
    assert np.isfinite(o_part).all() and np.isfinite(lse_part).all()
    C = oracle.attention._f64(wl.kv_range_bf16(w, "c", 0, 0, 0, 640, "cuda"))
    qb = oracle.attention._f64(q[0])
    sets = _gpu.shard_sets(w, 640)
    kept = np.concatenate([sets[1][:128], sets[1][192:]])
    for s_, idx in ((0, sets[0]), (1, kept)):
        Os, Ls = oracle.attend(qb, C[idx], C[idx][:, : w.dv], w.softmax_scale)
        _gpu.assert_close_O(o_part[s_, 0], Os, f"O_partial s={s_}")
        _gpu.assert_close_lse(lse_part[s_, 0], Ls, f"lse_partial s={s_}")


def test_mla_many_short_units():
    """Many requests with short, ragged histories: nearly every tile starts a new (request, shard)
    unit, so q (its shared-memory chunks and its half chunk in TMEM) is reloaded at almost every
    tile, and many shards are empty. Sharp queries make the weights peaked."""
    rng = np.random.default_rng(7)
    lens = [int(x) for x in rng.integers(1, 700, size=12)]
    lens[3] = 64  # exactly one page in one shard
    lens[5] = 1
    w = MLA.with_(B=12, S=max(lens), kvp=8)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens)
    assert cache.err_bits() == 0
    for sharp in (1.0, 8.0):
        q = wl.query(w, "cuda", scale_by=sharp)
        res = _run(cache, w, q)
        assert cache.err_bits() == 0
        _check(w, q, lens, res, f"many units x{sharp}", heads=list(range(0, 128, 9)))


def test_mla_batch_beyond_one_launch():
    """240 requests x 8 shards = 1,920 (request, shard) units, more than one launch keeps in shared
    memory: the partial runs as consecutive launches over request ranges, with the same results."""
    rng = np.random.default_rng(11)
    lens = [int(x) for x in rng.integers(1, 131, size=240)]
    w = MLA.with_(B=240, S=max(lens), kvp=8)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens)
    assert cache.err_bits() == 0
    q = wl.query(w, "cuda")
    res = _run(cache, w, q)
    assert cache.err_bits() == 0
    assert np.isfinite(res[2]).all() and np.isfinite(res[3]).all()
    _check(w, q, lens, res, "1920 units", heads=[0, 63, 127])
