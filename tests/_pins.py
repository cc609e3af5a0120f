"""Checks that pin the oracle to facts outside itself.

Each check takes the oracle functions it exercises as arguments, so ``test_oracle_mutations`` can
hand it a copy of the oracle with a planted mistake and confirm that the mistake is caught.
The checks use: closed forms of softmax attention, its invariances, an independent scalar brute
force on tiny inputs, PyTorch's fp64 CPU scaled_dot_product_attention / logsumexp as a library
special case, the pages' round-robin example, and the published NVFP4 element tables.
"""

from __future__ import annotations

import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    err = np.where(both_inf, 0.0, np.abs(a - b))
    assert np.all(np.isfinite(err)) and err.max(initial=0.0) <= tol, \
        f"{what}: max err {err.max(initial=0.0):.3e} > {tol:.1e}"


# ----------------------------------------------------------------------------------------------
# softmax attention


def brute_force_attend(q, K, V, scale):
    """Scalar-loop softmax attention with math.fsum, written independently of the oracle."""
    H, T, dv = len(q), len(K), len(V[0]) if len(V) else 0
    O, L = [], []
    for h in range(H):
        z = [scale * math.fsum(q[h][i] * K[t][i] for i in range(len(q[h]))) for t in range(T)]
        m = max(z)
        e = [math.exp(x - m) for x in z]
        s = math.fsum(e)
        O.append([math.fsum(e[t] * V[t][j] for t in range(T)) / s for j in range(dv)])
        L.append(m + math.log(s))
    return np.array(O), np.array(L)


def pin_brute_force(attend, seed=0):
    rng = np.random.default_rng(seed)
    for T in range(1, 9):
        for d, dv in ((1, 1), (3, 2), (4, 5)):
            q = rng.standard_normal((3, d))
            K = rng.standard_normal((T, d))
            V = rng.standard_normal((T, dv))
            sc = float(rng.uniform(0.1, 2.0))
            O, L = attend(q, K, V, sc)
            Ob, Lb = brute_force_attend(q.tolist(), K.tolist(), V.tolist(), sc)
            _close(O, Ob, 1e-12, f"brute force O (T={T})")
            _close(L, Lb, 1e-12, f"brute force lse (T={T})")


def pin_closed_forms(attend, seed=1):
    rng = np.random.default_rng(seed)
    d, dv, T = 16, 12, 37
    q = rng.standard_normal((4, d))
    K = rng.standard_normal((T, d))
    sc = 0.25
    # constant V -> O = V
    v = rng.standard_normal(dv)
    O, _ = attend(q, K, np.tile(v, (T, 1)), sc)
    _close(O, np.tile(v, (4, 1)), 1e-12, "constant V")
    # one token -> O = V_0, lse = z_0
    V1 = rng.standard_normal((1, dv))
    O, L = attend(q, K[:1], V1, sc)
    _close(O, np.tile(V1[0], (4, 1)), 1e-12, "single token O")
    _close(L, sc * (q @ K[0]), 1e-12, "single token lse")
    # q = 0 -> O = mean(V), lse = ln T exactly
    V = rng.standard_normal((T, dv))
    O, L = attend(np.zeros((2, d)), K, V, sc)
    _close(O, np.tile(V.mean(0), (2, 1)), 1e-12, "q=0 O")
    _close(L, np.full(2, math.log(T)), 1e-12, "q=0 lse")
    # identical keys -> lse = z + ln T, O = mean(V)
    k = rng.standard_normal(d)
    O, L = attend(q, np.tile(k, (T, 1)), V, sc)
    _close(L, sc * (q @ k) + math.log(T), 1e-12, "identical keys lse")
    _close(O, np.tile(V.mean(0), (4, 1)), 1e-12, "identical keys O")
    # a dominant key -> O -> its V, lse -> its logit (one-hot limit, exact to fp64 rounding)
    Kd = K.copy()
    Kd[5] = 60.0 * q[0] / np.linalg.norm(q[0])
    O, L = attend(q[:1], Kd, V, 1.0)
    _close(O[0], V[5], 1e-9, "dominant key O")
    # empty token set
    O, L = attend(q, K[:0], V[:0], sc)
    assert np.all(O == 0) and np.all(np.isneginf(L)), "empty set must give O=0, lse=-inf"


def pin_invariances(attend, seed=2):
    rng = np.random.default_rng(seed)
    d, dv, T = 8, 6, 50
    q = rng.standard_normal((5, d))
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, dv))
    sc = 0.7
    O, L = attend(q, K, V, sc)
    perm = rng.permutation(T)
    Op, Lp = attend(q, K[perm], V[perm], sc)
    _close(Op, O, 1e-12, "permutation O")
    _close(Lp, L, 1e-12, "permutation lse")
    u, c = rng.standard_normal(d), 1.7
    Os, Ls = attend(q, K + c * u, V, sc)
    _close(Os, O, 1e-11, "key shift O")
    _close(Ls, L + sc * c * (q @ u), 1e-11, "key shift lse")
    # adding a constant to V shifts O by it
    Ov, _ = attend(q, K, V + 3.0, sc)
    _close(Ov, O + 3.0, 1e-12, "value shift")


def pin_torch_sdpa(decode, seed=3):
    """Library special case: fp64 CPU scaled_dot_product_attention (GQA) and logsumexp."""
    g = torch.Generator().manual_seed(seed)
    for (B, Hq, Hkv, d, dv, S) in ((2, 8, 2, 16, 16, 33), (1, 16, 1, 24, 20, 17), (3, 4, 4, 8, 8, 5)):
        q = torch.randn(B, Hq, d, generator=g, dtype=torch.float64)
        K = torch.randn(B, S, Hkv, d, generator=g, dtype=torch.float64)
        V = torch.randn(B, S, Hkv, dv, generator=g, dtype=torch.float64)
        sc = 1.0 / math.sqrt(d)
        O, L = decode(q, K, V, [S] * B, sc)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, :, None, :], K.transpose(1, 2), V.transpose(1, 2), scale=sc, enable_gqa=True)[:, :, 0]
        G = Hq // Hkv
        Kx = K.repeat_interleave(G, dim=2)  # [B, S, Hq, d], head h -> KV head h // G
        z = torch.einsum("bhd,bshd->bhs", q, Kx) * sc
        _close(O, ref.numpy(), 1e-12, "SDPA O")
        _close(L, torch.logsumexp(z, -1).numpy(), 1e-12, "logsumexp lse")


# ----------------------------------------------------------------------------------------------
# combine


def pin_combine_identity(attend, combine, shard_tokens, seed=4):
    """Sharded attention + combine == unsharded attention, for any partition of the tokens."""
    rng = np.random.default_rng(seed)
    d, dv = 16, 16
    for trial in range(30):
        T = int(rng.integers(1, 300))
        P = int(rng.integers(1, 17))
        q = rng.standard_normal((6, d)) * (3.0 if trial % 3 == 0 else 1.0)
        K = rng.standard_normal((T, d))
        V = rng.standard_normal((T, dv))
        sc = 1 / math.sqrt(d)
        O, L = attend(q, K, V, sc)
        if trial % 3 == 0:
            parts = np.array_split(rng.permutation(T), P)  # random partition
        elif trial % 3 == 1:
            parts = shard_tokens(T, P, "rr", 16)
        else:
            parts = shard_tokens(T, P, "contig", chunk=-(-T // P))
        Os, Ls = zip(*[attend(q, K[p], V[p], sc) for p in parts])
        Oc, Lc = combine(np.stack(Os), np.stack(Ls))
        _close(Oc, O, 1e-12 * max(1.0, np.abs(O).max()), f"combine identity O (P={P}, T={T})")
        _close(Lc, L, 1e-12 * max(1.0, np.abs(L).max()), f"combine identity lse (P={P}, T={T})")
    # one shard: identity
    Oc, Lc = combine(O[None], L[None])
    _close(Oc, O, 0.0, "P=1 O")
    _close(Lc, L, 0.0, "P=1 lse")
    # empty shards carry no weight; all-empty gives O=0, lse=-inf
    Oe = np.zeros_like(O)
    Le = np.full_like(L, -np.inf)
    Oc, Lc = combine(np.stack([Oe, O, Oe]), np.stack([Le, L, Le]))
    _close(Oc, O, 1e-15, "empty shards O")
    _close(Lc, L, 1e-15, "empty shards lse")
    Oc, Lc = combine(np.stack([Oe, Oe]), np.stack([Le, Le]))
    assert np.all(Oc == 0) and np.all(np.isneginf(Lc)), "all-empty combine"


# ----------------------------------------------------------------------------------------------
# layout


def pin_layout(rr_place, contig_place, shard_tokens, shard_lens, page_slot):
    for t, s in _golden_rows("rr16_blog_example.txt"):
        for P in (2, 3, 4, 8):
            assert rr_place(int(t), P, 16)[0] == int(s), f"blog example t={t} P={P}"
    want = {0: [], 1: [], 2: []}
    for s, a, b in _golden_rows("rr16_p3_s100.txt"):
        want[int(s)].extend(range(int(a), int(b) + 1))
    got = shard_tokens(100, 3, "rr", 16)
    for s in range(3):
        assert list(got[s]) == want[s], f"P=3 S=100 shard {s}"
    assert shard_lens(100, 3, "rr", 16) == [len(want[s]) for s in range(3)]
    for P in (1, 2, 3, 8):
        for S in (1, 15, 16, 17, 200, 1000):
            parts = shard_tokens(S, P, "rr", 16)
            flat = np.sort(np.concatenate(parts))
            assert np.array_equal(flat, np.arange(S)), "each token exactly once"
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 16, "round-robin keeps shards within one block"
            for s, p in enumerate(parts):
                for l_, t in enumerate(p):
                    assert rr_place(int(t), P, 16) == (s, l_)
    assert contig_place(1500, 1024) == (1, 476)
    parts = shard_tokens(4096, 4, "contig", chunk=1024)
    assert [int(p[0]) for p in parts] == [0, 1024, 2048, 3072] and all(len(p) == 1024 for p in parts)
    assert page_slot(0) == (0, 0) and page_slot(63) == (0, 63) and page_slot(64) == (1, 0)
    assert page_slot(130, 64) == (2, 2)


# ----------------------------------------------------------------------------------------------
# NVFP4


def pin_nvfp4(e2m1_value, e4m3_value, nvfp4_dequant):
    for code, val in _golden_rows("e2m1_ocp_mx.txt"):
        assert e2m1_value(int(code)) == float(val), f"e2m1 code {code}"
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        a, b = e4m3_value(c), float(lib[c])
        assert (math.isnan(a) and math.isnan(b)) or a == b, f"e4m3 code {c}: {a} vs {b}"
    assert e4m3_value(0x7E) == 448.0 and e4m3_value(0x01) == 2.0 ** -9
    # packing: element 2i in the low nibble; scale j covers elements 16j..16j+15
    codes = np.zeros((1, 16), dtype=np.uint8)
    codes[0, 0] = 0x72  # element 0 -> code 2 (1.0), element 1 -> code 7 (6.0)
    codes[0, 8] = 0x0B  # element 16 -> code 11 (-1.5)
    codes[0, 5] = 0x04  # element 10 -> code 4 (2.0), still in scale block 0
    codes[0, 15] = 0x50  # element 31 -> code 5 (3.0), scale block 1
    scales = np.zeros((1, 2), dtype=np.uint8)
    scales[0, 0] = 0x38  # 1.0
    scales[0, 1] = 0x40  # 2.0
    x = nvfp4_dequant(codes, scales)
    assert x.shape == (1, 32)
    assert x[0, 0] == 1.0 and x[0, 1] == 6.0 and x[0, 16] == -3.0 and x[0, 2] == 0.0
    assert x[0, 10] == 2.0 and x[0, 11] == 0.0 and x[0, 31] == 6.0 and x[0, 30] == 0.0


def pin_nvfp4_encode(nvfp4_encode, seed=6):
    """The quantiser: hand-derived blocks (every E2M1 tie, saturation, the 448 clamp, scale 0,
    a subnormal scale, E4M3 scale ties), the scale against torch's float8_e4m3fn rounding, the
    per-element error bound, and agreement with the input generator's separate encoder."""
    for name, vals, sc, codes in (
            [p.strip() for p in " ".join(r).split("|")] for r in _golden_rows("nvfp4_encode_cases.txt")):
        x = np.array([float(v) for v in vals.split()], dtype=np.float32)[None]
        c, s = nvfp4_encode(x)
        assert int(np.asarray(s)[0, 0]) == int(sc, 16), f"{name}: scale"
        assert [int(v) for v in np.asarray(c)[0]] == [int(b, 16) for b in codes.split()], name
    g = torch.Generator().manual_seed(seed)
    # magnitudes over many binades, including blocks whose absmax / 6 exceeds 448 or underflows
    x = torch.randn(512, 64, generator=g) * torch.exp2(torch.randint(-14, 13, (512, 1), generator=g).float())
    x[0] = 0.0
    c, s = nvfp4_encode(x)
    c, s = np.asarray(c), np.asarray(s)
    amax = x.reshape(512, 4, 16).abs().amax(-1)
    r = (amax / 6.0).clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, r), "scale differs from torch's E4M3 rounding"
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    half_gap = np.array([0.25, 0.25, 0.25, 0.25, 0.5, 0.5, 1.0, 1.0])  # max error per magnitude
    lo = c & 0xF
    hi = c >> 4
    code = np.stack([lo, hi], -1).reshape(512, 64)
    sign = np.where(code & 8, -1.0, 1.0)
    mag_i = code & 7
    sd = np.repeat(torch.from_numpy(s.copy()).view(torch.float8_e4m3fn).double().numpy(), 16,
                   axis=1)
    xd = x.double().numpy()
    y = np.where(sd > 0, xd / np.where(sd > 0, sd, 1.0), xd)
    dec = sign * mags[mag_i]
    sat = np.abs(y) > 6.0
    assert np.all(np.abs(dec[~sat] - y[~sat]) <= half_gap[mag_i][~sat] * (1 + 1e-6) + 1e-12)
    assert np.all(np.abs(dec[sat]) == 6.0) and np.all(np.sign(dec[sat]) == np.sign(y[sat]))
    assert not np.any((mag_i == 0) & (code & 8)), "a zero magnitude carries a sign"
    # an independent encoder (the input generator's, thresholds in torch) gives the same bytes
    import workloads

    c2, s2 = workloads.nvfp4_encode(x)
    assert np.array_equal(c, c2.numpy()) and np.array_equal(s, s2.numpy())
