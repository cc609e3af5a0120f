"""fp64 reference for decode attention, its sequence-sharded partials and the LSE combine.

TEST INFRASTRUCTURE (see the package docstring): only tests/, smoke() and bench.py's CPU legs use it.

Everything is the plain definition, two passes, no online rescaling, no blocking:

    z_t   = scale * <q, K_t>                   for every history token t of the request
    m     = max_t z_t
    w_t   = exp(z_t - m)
    O     = sum_t w_t V_t / sum_t w_t
    lse   = m + ln sum_t w_t                   (natural log)

Inputs are whatever dtype the caller has; they are converted to fp64 exactly (bf16 -> fp64 and the
NVFP4 decode in ``oracle.nvfp4`` are exact), so the only rounding is fp64's.
"""

from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: go through fp64 on the CPU (exact for bf16/f16/f32)
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attend(q, K, V, scale: float):
    """Attention of H query rows against one token set.

    q [H, d], K [T, d], V [T, dv] -> (O [H, dv], lse [H]).
    Source: paper summary (fdeinterviews.com), paragraph on KV parallelism -- a shard's partial output
    is the softmax-weighted value average over its slice, reported with the slice's log-sum-exp.
    An empty token set (T = 0) gives O = 0 and lse = -inf: the shard holds nothing, so it must carry
    zero weight in the combine.
    """
    q, K, V = _f64(q), _f64(K), _f64(V)
    H, T, dv = q.shape[0], K.shape[0], V.shape[1]
    if T == 0:
        return np.zeros((H, dv)), np.full(H, -np.inf)
    z = scale * (q @ K.T)  # [H, T] logits
    m = z.max(axis=1)
    w = np.exp(z - m[:, None])
    den = w.sum(axis=1)
    O = (w @ V) / den[:, None]
    lse = m + np.log(den)
    return O, lse


def _group_of(h: int, num_q_heads: int, num_kv_heads: int) -> int:
    """GQA head mapping: contiguous groups of G = Hq/Hkv query heads share one KV head.

    The pages give only the head counts (Q = 128 query heads against K = 8 KV heads in the paper
    review's "state of the art" list, and MLA as "effectively one" KV head in the paper summary's
    tensor-parallelism paragraph); contiguous grouping is the plain reading.
    """
    return h // (num_q_heads // num_kv_heads)


def decode(q, K, V, seq_lens, scale: float):
    """Unsharded decode attention for a batch.

    q [B, Hq, d]; K [B, S_max, Hkv, d]; V [B, S_max, Hkv, dv] (logical, token-major history);
    seq_lens [B]. Returns O [B, Hq, dv] and lse [B, Hq].
    For MLA pass Hkv = 1, K = the 576-wide latent and V = its first 512 columns.
    """
    q = _f64(q)
    B, Hq, _ = q.shape
    Hkv, dv = K.shape[2], V.shape[3]
    O = np.zeros((B, Hq, dv))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        S = int(seq_lens[b])
        for h in range(Hq):
            k = _group_of(h, Hq, Hkv)
            o, l_ = attend(q[b, h : h + 1], K[b, :S, k], V[b, :S, k], scale)
            O[b, h], lse[b, h] = o[0], l_[0]
    return O, lse


def partial(q, K, V, token_sets, scale: float):
    """Per-shard partial attention.

    token_sets[b][s] lists the global positions t that KVP shard s holds for request b.
    Returns O_s [P, B, Hq, dv] (each shard's output normalised over its own tokens) and
    lse_s [P, B, Hq] (natural log; -inf for an empty shard).
    Source: paper summary (fdeinterviews.com), paragraph on KV parallelism.
    """
    q = _f64(q)
    B, Hq, _ = q.shape
    Hkv, dv = K.shape[2], V.shape[3]
    P = len(token_sets[0])
    O_s = np.zeros((P, B, Hq, dv))
    lse_s = np.full((P, B, Hq), -np.inf)
    for b in range(B):
        for s in range(P):
            idx = np.asarray(token_sets[b][s], dtype=np.int64)
            for h in range(Hq):
                k = _group_of(h, Hq, Hkv)
                o, l_ = attend(q[b, h : h + 1], _f64(K[b, idx, k]).reshape(len(idx), -1),
                               _f64(V[b, idx, k]).reshape(len(idx), -1), scale)
                O_s[s, b, h], lse_s[s, b, h] = o[0], l_[0]
    return O_s, lse_s


def combine(O_s, lse_s):
    """LSE-rescaling combine of normalised per-shard partials.

    O_s [P, ..., dv], lse_s [P, ...] -> O [..., dv], lse [...].
    Source: paper review (jaehun.me), "Prompt 1.3.2 -- The Secret Weapon", boxed equation: the full
    output is the sum of the partial outputs weighted by e^{lse_i}, divided by the sum of e^{lse_i}.
    That form is exact only for partials normalised over their own slice, which is how ``partial``
    returns them. Written with the largest lse factored out:

        M   = max_s lse_s
        LSE = M + ln sum_s exp(lse_s - M)
        O   = sum_s exp(lse_s - LSE) * O_s

    Shards with lse = -inf contribute zero weight. If every shard is empty the result is O = 0 and
    LSE = -inf.
    """
    O_s, lse_s = _f64(O_s), _f64(lse_s)
    M = lse_s.max(axis=0)
    alive = np.isfinite(M)
    M0 = np.where(alive, M, 0.0)
    w = np.exp(lse_s - M0)  # exp(-inf) = 0 for empty shards
    den = w.sum(axis=0)
    safe_den = np.where(alive, den, 1.0)
    LSE = np.where(alive, M0 + np.log(safe_den), -np.inf)
    O = (w[..., None] * O_s).sum(axis=0) / safe_den[..., None]
    O = np.where(alive[..., None], O, 0.0)
    return O, LSE
