"""Helpers for the GPU tests: build a cache for a workload, fill it through the library's append,
and fetch the same seeded inputs for the oracle."""

from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as wl

TOL_O = 1e-2  # max-abs error on O and O_partial (bf16 / NVFP4 inputs, fp32 accumulation)
TOL_LSE = 1e-3  # max-abs error on the natural-log LSE
TOL_REL = 1e-2  # ||O - O*|| / ||O*||, the check that stays meaningful when |O| is small at long S


def hx():
    import long_context_decode_helix_b200 as m

    return m


def make_cache(w: wl.Workload, S_cap: int | None = None, shuffle: bool = True, device="cuda"):
    m = hx()
    pt, n = wl.page_table(w, S_cap, shuffle)
    return m.KVCache(
        m.ATTN_MLA if w.kind == "mla" else m.ATTN_GQA,
        m.KV_NVFP4 if w.kv_dtype == "nvfp4" else m.KV_BF16,
        m.LAYOUT_RR if w.layout == "rr" else m.LAYOUT_CONTIG,
        w.kvp, w.B, w.Hkv, w.d, w.dv, pt.shape[2], page_tokens=w.page_tokens,
        rr_block=w.rr_block, contig_chunk=w.contig_chunk, page_table=pt, num_pages=n, device=device)


def new_rows(w: wl.Workload, t0: int, t1: int, device="cuda"):
    """The append arguments for history positions [t0, t1) of every request."""
    return wl.append_rows(w, t0, t1, device)


def fill(cache, w: wl.Workload, lens, chunk: int = 32768, device="cuda"):
    """Append every request's history [0, lens[b]) through helix_kv_append, ragged by n_valid."""
    m = hx()
    S_max = max(lens)
    for t0 in range(0, S_max, chunk):
        n = min(chunk, S_max - t0)
        nv = torch.tensor([min(max(L - t0, 0), n) for L in lens], dtype=torch.int32, device=device)
        m.append(cache, **new_rows(w, t0, t0 + n, device), n_valid=nv)
    torch.cuda.synchronize()


def oracle_kv(w: wl.Workload, b: int, h: int, S: int, device="cuda"):
    """fp64 K [S, d] and V [S, dv] of one (request, KV head), decoded exactly from what the GPU got."""
    if w.kind == "mla":
        c = oracle.attention._f64(wl.kv_range_bf16(w, "c", b, 0, 0, S, device))
        return c, c[:, : w.dv]
    if w.kv_dtype == "nvfp4":
        kc, ks = wl.kv_range_nvfp4(w, "k", b, h, 0, S, device)
        vc, vs = wl.kv_range_nvfp4(w, "v", b, h, 0, S, device)
        return oracle.nvfp4_dequant(kc, ks), oracle.nvfp4_dequant(vc, vs)
    return (oracle.attention._f64(wl.kv_range_bf16(w, "k", b, h, 0, S, device)),
            oracle.attention._f64(wl.kv_range_bf16(w, "v", b, h, 0, S, device)))


def shard_sets(w: wl.Workload, S: int):
    return oracle.shard_tokens(S, w.kvp, w.layout, w.rr_block, w.contig_chunk)


def oracle_head_group(w, q, b, h, S, device="cuda"):
    """Oracle for the G query heads of KV head h of request b: per-shard (O_s, lse_s) and the
    unsharded (O, lse)."""
    K, V = oracle_kv(w, b, h, S, device)
    qg = oracle.attention._f64(q[b, h * w.G:(h + 1) * w.G])
    O, L = oracle.attend(qg, K, V, w.softmax_scale)
    parts = [oracle.attend(qg, K[idx], V[idx], w.softmax_scale) for idx in shard_sets(w, S)]
    return O, L, np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts])


def assert_close_O(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert err.max(initial=0) <= TOL_O, f"{what}: max-abs {err.max():.3e} > {TOL_O}"
    nrm = np.linalg.norm(want)
    if nrm > 0:
        rel = np.linalg.norm(got - want) / nrm
        assert rel <= TOL_REL, f"{what}: relative {rel:.3e} > {TOL_REL}"


def assert_close_lse(got, want, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both = np.isneginf(got) & np.isneginf(want)
    with np.errstate(invalid="ignore"):
        err = np.where(both, 0.0, np.abs(got - want))
    assert np.all(np.isfinite(err)), f"{what}: -inf mismatch"
    assert err.max(initial=0) <= TOL_LSE, f"{what}: max-abs {err.max():.3e} > {TOL_LSE}"
