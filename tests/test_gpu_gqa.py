"""GQA decode attention on the GPU against the fp64 oracle (append -> partial -> combine).

Tolerances: max-abs 1e-2 on O and O_partial, 1e-3 on LSE, and relative L2 error 1e-2 on O.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu


def _run(cache, w, q):
    hx = _gpu.hx()
    o_part, lse_part = hx.partial(cache, q, w.softmax_scale)
    out, lse = hx.combine(o_part, lse_part, out_dtype=torch.float32)
    torch.cuda.synchronize()
    return o_part.cpu().numpy(), lse_part.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def _check_all_heads(w, q, lens, res, label):
    o_part, lse_part, out, lse = res
    for b in range(w.B):
        for h in range(w.Hkv):
            O, L, Os, Ls = _gpu.oracle_head_group(w, q, b, h, lens[b])
            hs = slice(h * w.G, (h + 1) * w.G)
            _gpu.assert_close_O(out[b, hs], O, f"{label} O b={b} h={h}")
            _gpu.assert_close_lse(lse[b, hs], L, f"{label} LSE b={b} h={h}")
            _gpu.assert_close_O(o_part[:, b, hs], Os, f"{label} O_partial b={b} h={h}")
            _gpu.assert_close_lse(lse_part[:, b, hs], Ls, f"{label} lse_partial b={b} h={h}")


SMALL = {
    # the tiny workload itself: B=1, Hq=8, Hkv=2, d=64, S=4096, four contiguous shards
    "tiny": (wl.WORKLOADS["tiny_gqa"], [4096]),
    # round-robin-16 over 8 shards, G=16, ragged lengths: one token, a partial page, several tiles
    "rr_g16_ragged": (wl.WORKLOADS["gqa_s128k"].with_(B=3, Hq=48, Hkv=3, S=3000),
                      [3000, 1, 77]),
    # more shards than 16-token blocks: most shards empty for the short requests
    "rr_empty_shards": (wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=16, Hkv=2, S=40), [40, 17]),
    # G=1 (multi-head), d=64, contiguous layout with a ragged last shard
    "contig_mha": (wl.WORKLOADS["tiny_gqa"].with_(B=2, Hq=4, Hkv=4, S=1000, kvp=3), [1000, 999]),
    # G=4, d=128, a long enough history that several CTAs split each unit
    "rr_split_units": (wl.WORKLOADS["gqa_s128k"].with_(B=1, Hq=8, Hkv=2, S=70000, kvp=2),
                       [70000]),
}


NVFP4 = wl.WORKLOADS["gqa_nvfp4_s1m"]
SMALL.update({
    # NVFP4 KV: ragged lengths with G=16, empty shards, and units split across CTAs
    "nvfp4_rr_ragged": (NVFP4.with_(B=3, Hq=48, Hkv=3, S=3000), [3000, 1, 77]),
    "nvfp4_empty_shards": (NVFP4.with_(B=2, Hq=16, Hkv=2, S=40), [40, 17]),
    "nvfp4_split_units": (NVFP4.with_(B=1, Hq=8, Hkv=2, S=70000, kvp=2), [70000]),
    "nvfp4_g4": (NVFP4.with_(B=2, Hq=16, Hkv=4, S=2500, kvp=3), [2500, 1300]),
})


@pytest.mark.parametrize("name", sorted(SMALL))
def test_gqa_small(name):
    w, lens = SMALL[name]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=1024)
    assert cache.err_bits() == 0
    q = wl.query(w, "cuda")
    _check_all_heads(w, q, lens, _run(cache, w, q), name)


def test_gqa_nvfp4_sharp():
    """NVFP4 KV with a sharp query (q x 8): near one-hot softmax, |O| of order |V|."""
    w = NVFP4.with_(B=2, Hq=32, Hkv=2, S=5000)
    lens = [5000, 4321]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=2048)
    q = wl.query(w, "cuda", scale_by=8.0)
    res = _run(cache, w, q)
    _check_all_heads(w, q, lens, res, "nvfp4 sharp")
    assert np.abs(res[2]).max() > 0.3


@pytest.mark.parametrize("kind", ["sharp", "needle", "shift"])
def test_gqa_structured_inputs(kind):
    """Inputs that make |O| large, so the absolute tolerance is not vacuous."""
    w = wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=32, Hkv=2, S=5000)
    lens = [5000, 4321]
    cache = _gpu.make_cache(w)
    q = wl.query(w, "cuda", scale_by=8.0 if kind == "sharp" else 1.0)
    rows = _gpu.new_rows(w, 0, w.S)
    if kind == "needle":  # a few keys aligned with the group's mean query direction
        for b in range(w.B):
            for h in range(w.Hkv):
                qd = q[b, h * w.G:(h + 1) * w.G].float().mean(0)
                for t in (3, 1777, 4000):
                    rows["k_new"][b, t, h] = (6.0 * qd / qd.norm()).to(torch.bfloat16)
    if kind == "shift":  # the same offset added to every key
        u = torch.randn(w.d, generator=torch.Generator().manual_seed(5)).cuda()
        rows["k_new"] = (rows["k_new"].float() + 2.0 * u).to(torch.bfloat16)
    hx = _gpu.hx()
    hx.append(cache, rows["k_new"], rows["v_new"],
              n_valid=torch.tensor(lens, dtype=torch.int32, device="cuda"))
    o_part, lse_part, out, lse = _run(cache, w, q)
    K = rows["k_new"].cpu()
    V = rows["v_new"].cpu()
    O, L = oracle.decode(q, K, V, lens, w.softmax_scale)
    _gpu.assert_close_O(out, O, kind)
    _gpu.assert_close_lse(lse, L, kind)
    if kind == "sharp":
        assert np.abs(O).max() > 0.5  # the check is not vacuous


def test_gqa_decode_loop():
    """Token-by-token decode: every step appends one token and attends over the grown history."""
    w = wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=16, Hkv=1, S=2000)
    lens0 = [1990, 1500]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens0, chunk=512)
    hx = _gpu.hx()
    q = wl.query(w, "cuda")
    allk = _gpu.new_rows(w, 0, w.S)
    for step in range(5):
        nv = torch.ones(w.B, dtype=torch.int32, device="cuda")
        # request b's next row is its position lens0[b] + step
        k1 = torch.stack([allk["k_new"][b, lens0[b] + step] for b in range(w.B)])[:, None]
        v1 = torch.stack([allk["v_new"][b, lens0[b] + step] for b in range(w.B)])[:, None]
        out, lse = hx.decode_step(cache, q, k1.contiguous(), v1.contiguous(), w.softmax_scale)
        torch.cuda.synchronize()
        lens = [L + step + 1 for L in lens0]
        O, L = oracle.decode(q, allk["k_new"].cpu(), allk["v_new"].cpu(), lens, w.softmax_scale)
        _gpu.assert_close_O(out.float().cpu().numpy(), O, f"step {step}")
        _gpu.assert_close_lse(lse.cpu().numpy(), L, f"step {step}")
    assert cache["seq_lens"].tolist() == [L + 5 for L in lens0]
    want = [oracle.shard_lens(L + 5, w.kvp, "rr", 16) for L in lens0]
    assert cache["shard_lens"].t().tolist() == want


def test_gqa_repeat_is_deterministic_and_tickets_reset():
    """Two calls in a row give bit-identical partials (the workspace tickets return to zero)."""
    w = wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=32, Hkv=2, S=20000)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, [20000, 13333], chunk=4096)
    q = wl.query(w, "cuda")
    a = _run(cache, w, q)
    b = _run(cache, w, q)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    ws = cache.workspace(w.Hq)
    assert int(ws[: 4 * w.B * w.Hkv * w.kvp].view(torch.int32).abs().sum()) == 0


@pytest.mark.parametrize("kv_dtype", ["bf16", "nvfp4"])
def test_gqa_repeat_variable_lengths_bit_identical(kv_dtype):
    """Ragged lengths (a partial last page in every unit), many split units, several calls: the
    results must not depend on the order in which pages land or warps finish."""
    base = wl.WORKLOADS["gqa_s1m_var" if kv_dtype == "bf16" else "gqa_nvfp4_s1m"]
    w = base.with_(B=8, Hq=32, Hkv=2, S=150000, S_min=None)
    g = torch.Generator().manual_seed(11)
    lens = [int(x) for x in torch.randint(40000, 150001, (w.B,), generator=g)]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=16384)
    q = wl.query(w, "cuda")
    first = _run(cache, w, q)
    for _ in range(3):
        again = _run(cache, w, q)
        for x, y in zip(first, again):
            assert np.array_equal(x, y)
    for b, h in ((int(np.argmin(lens)), 0), (int(np.argmax(lens)), 1)):
        O, L, Os, Ls = _gpu.oracle_head_group(w, q, b, h, lens[b])
        hs = slice(h * w.G, (h + 1) * w.G)
        _gpu.assert_close_O(first[2][b, hs], O, f"O b={b}")
        _gpu.assert_close_lse(first[3][b, hs], L, f"LSE b={b}")


@pytest.mark.parametrize("kv_dtype", ["bf16", "nvfp4"])
def test_gqa_bad_page_id_sets_error_and_skips(kv_dtype):
    """A page id outside the pool sets the device error bit, and that page's 64 tokens are left out
    of its shard; the rest of the shard is still attended exactly."""
    base = wl.WORKLOADS["gqa_s128k" if kv_dtype == "bf16" else "gqa_nvfp4_s1m"]
    w = base.with_(B=1, Hq=16, Hkv=1, S=640, kvp=2)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, [640])
    cache.page_table[1, 0, 2] = 10 ** 6  # beyond the pool: local tokens 128..191 of shard 1
    cache.clear_errors()
    q = wl.query(w, "cuda")
    o_part, lse_part, _, _ = _run(cache, w, q)
    assert cache.err_bits() & _gpu.hx().DEVERR_PAGE_ID
    K, V = _gpu.oracle_kv(w, 0, 0, 640)
    qg = oracle.attention._f64(q[0, : w.G])
    sets = _gpu.shard_sets(w, 640)
    kept = np.concatenate([sets[1][:128], sets[1][192:]])
    for s_, idx in ((0, sets[0]), (1, kept)):
        Os, Ls = oracle.attend(qg, K[idx], V[idx], w.softmax_scale)
        _gpu.assert_close_O(o_part[s_, 0, : w.G], Os, f"O_partial s={s_}")
        _gpu.assert_close_lse(lse_part[s_, 0, : w.G], Ls, f"lse_partial s={s_}")


# ---------------------------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times; sampled head groups


def _sampled(w, lens, samples):
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens)
    assert cache.err_bits() == 0
    q = wl.query(w, "cuda")
    hx = _gpu.hx()
    o_part, lse_part = hx.partial(cache, q, w.softmax_scale)
    out, lse = hx.combine(o_part, lse_part)  # bf16 output, as the benchmark step produces it
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b, h in samples:
        O, L, Os, Ls = _gpu.oracle_head_group(w, q, b, h, lens[b])
        hs = slice(h * w.G, (h + 1) * w.G)
        _gpu.assert_close_O(out[b, hs].float().cpu().numpy(), O, f"O b={b} h={h}")
        _gpu.assert_close_lse(lse[b, hs].cpu().numpy(), L, f"LSE b={b} h={h}")
        _gpu.assert_close_O(o_part[:, b, hs].cpu().numpy(), Os, f"O_partial b={b} h={h}")
        _gpu.assert_close_lse(lse_part[:, b, hs].cpu().numpy(), Ls, f"lse_partial b={b} h={h}")
    # properties that hold at any size: LSE >= max over shards, O within the V range
    lse_cpu = lse.cpu()
    assert torch.all(lse_cpu + 1e-4 >= lse_part.max(0).values.cpu())
    del cache
    torch.cuda.empty_cache()


def test_gqa_full_128k_sampled():
    w = wl.WORKLOADS["gqa_s128k"]
    _sampled(w, wl.seq_lens(w), [(0, 0), (7, 7), (3, 5)])


def test_gqa_full_1m_sampled():
    w = wl.WORKLOADS["gqa_s1m"]
    _sampled(w, wl.seq_lens(w), [(0, 0), (6, 3)])


def test_gqa_nvfp4_full_1m_sampled():
    w = wl.WORKLOADS["gqa_nvfp4_s1m"]
    _sampled(w, wl.seq_lens(w), [(0, 0), (5, 6)])


def test_gqa_full_1m_variable_sampled():
    w = wl.WORKLOADS["gqa_s1m_var"]
    lens = wl.seq_lens(w)
    _sampled(w, lens, [(int(np.argmin(lens)), 1), (int(np.argmax(lens)), 6)])
