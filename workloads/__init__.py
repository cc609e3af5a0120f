"""Seeded synthetic workloads for KV-parallel decode attention: shapes, inputs and byte counts.

This module is shared by the tests, ``bench.py`` and ``smoke()``. It holds no attention, layout or
combine arithmetic (that lives in the CUDA library and, separately, in the test oracle); it only
draws inputs and counts the bytes a step must move.

Shapes follow the models the pages evaluate -- Llama-405B-like GQA with 128 query heads and 8 KV
heads, and DeepSeek-R1-like MLA with one shared latent head -- at a 1M-token context (paper review,
jaehun.me, "Prompt 1.4.1 -- Key Results with Metrics", benchmarks and environment). No weights or
datasets are involved: q, K and V are i.i.d. N(0, 1) draws rounded to bf16 (or encoded to NVFP4).

Reproducibility: every block of GEN_BLOCK tokens of every (request, KV head) stream is drawn from its
own torch generator, keyed by splitmix64 over (workload seed, tensor id, request, head, block). Any
token range can therefore be regenerated without materialising the whole history (a 1M-token bf16
history is 32 GiB). Generation is deterministic per device; tests draw on one device and feed the
same tensors to both sides.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

GEN_BLOCK = 4096
_MASK64 = (1 << 64) - 1
_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "c": 4, "lens": 5, "pages": 6, "knew": 7, "vnew": 8, "cnew": 9}


def splitmix64(x: int) -> int:
    """SplitMix64 finaliser (Steele, Lea and Flood, 2014): a published 64-bit mixing function."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def stream_seed(seed: int, *keys: int) -> int:
    h = splitmix64(seed)
    for k in keys:
        h = splitmix64(h ^ (int(k) & _MASK64))
    return h & ((1 << 63) - 1)


def _gen(device, seed: int, *keys) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, *keys))
    return g


@dataclass(frozen=True)
class Workload:
    """One decode-attention layer step: B requests, one new query token each."""

    name: str
    kind: str  # "gqa" or "mla"
    kv_dtype: str  # "bf16" or "nvfp4"
    B: int
    Hq: int
    Hkv: int
    d: int  # K width (576 for MLA)
    dv: int  # V width (d for GQA, 512 for MLA)
    S: int  # context length per request (the maximum when lengths vary)
    kvp: int
    layout: str  # "rr" (round-robin blocks) or "contig"
    seed: int
    S_min: int | None = None  # lengths drawn uniformly in [S_min, S] when set
    rr_block: int = 16
    page_tokens: int = 64
    # the final length the contiguous layout is sized for (C = ceil(S_final / P)); None = S. A
    # decode loop that appends past S needs it, or the new tokens would fall off the last shard.
    S_final: int | None = None

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def contig_chunk(self) -> int:
        return -(-(self.S if self.S_final is None else self.S_final) // self.kvp)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # configs in the order the workload list gives them; seed = 1000 + position
    "tiny_gqa": Workload("tiny_gqa", "gqa", "bf16", B=1, Hq=8, Hkv=2, d=64, dv=64, S=4096, kvp=4,
                         layout="contig", seed=1001),
    "gqa_s128k": Workload("gqa_s128k", "gqa", "bf16", B=8, Hq=128, Hkv=8, d=128, dv=128, S=131072,
                          kvp=8, layout="rr", seed=1002),
    "gqa_s1m": Workload("gqa_s1m", "gqa", "bf16", B=8, Hq=128, Hkv=8, d=128, dv=128, S=1 << 20,
                        kvp=8, layout="rr", seed=1003),
    "gqa_s1m_var": Workload("gqa_s1m_var", "gqa", "bf16", B=8, Hq=128, Hkv=8, d=128, dv=128,
                            S=1 << 20, S_min=1 << 19, kvp=8, layout="rr", seed=1003),
    "gqa_nvfp4_s1m": Workload("gqa_nvfp4_s1m", "gqa", "nvfp4", B=8, Hq=128, Hkv=8, d=128, dv=128,
                              S=1 << 20, kvp=8, layout="rr", seed=1004),
    "mla_s1m": Workload("mla_s1m", "mla", "bf16", B=8, Hq=128, Hkv=1, d=576, dv=512, S=1 << 20,
                        kvp=8, layout="rr", seed=1005),
}


# ----------------------------------------------------------------------------------------------
# inputs


def seq_lens(w: Workload) -> list[int]:
    """Per-request context length: S, or uniform integers in [S_min, S] drawn from the seed."""
    if w.S_min is None:
        return [w.S] * w.B
    g = _gen("cpu", w.seed, _TENSOR_IDS["lens"])
    return [int(x) for x in torch.randint(w.S_min, w.S + 1, (w.B,), generator=g)]


def normal(shape, seed: int, *keys, device="cpu") -> torch.Tensor:
    """fp32 N(0,1) draw from a keyed generator."""
    return torch.randn(shape, generator=_gen(device, seed, *keys), device=device,
                       dtype=torch.float32)


def query(w: Workload, device="cpu", scale_by: float = 1.0) -> torch.Tensor:
    """q [B, Hq, d] bf16 (rounded to nearest even from fp32 N(0,1), optionally multiplied first)."""
    x = normal((w.B, w.Hq, w.d), w.seed, _TENSOR_IDS["q"], device=device)
    return (x * scale_by).to(torch.bfloat16)


def kv_block_f32(w: Workload, which: str, b: int, h: int, blk: int, device="cpu") -> torch.Tensor:
    """fp32 N(0,1) values of tokens [blk*GEN_BLOCK, (blk+1)*GEN_BLOCK) of one (request, head)."""
    return normal((GEN_BLOCK, w.d), w.seed, _TENSOR_IDS[which], b, h, blk, device=device)


def kv_range_f32(w: Workload, which: str, b: int, h: int, t0: int, t1: int, device="cpu"):
    """fp32 values of tokens [t0, t1) of one (request, head) stream: [t1 - t0, d]."""
    if t1 <= t0:
        return torch.empty((0, w.d), dtype=torch.float32, device=device)
    parts = []
    for blk in range(t0 // GEN_BLOCK, (t1 - 1) // GEN_BLOCK + 1):
        x = kv_block_f32(w, which, b, h, blk, device)
        lo = max(t0 - blk * GEN_BLOCK, 0)
        hi = min(t1 - blk * GEN_BLOCK, GEN_BLOCK)
        parts.append(x[lo:hi])
    return torch.cat(parts, 0)


def kv_range_bf16(w, which, b, h, t0, t1, device="cpu"):
    return kv_range_f32(w, which, b, h, t0, t1, device).to(torch.bfloat16)


def kv_tokens(w: Workload, which: str, b: int, t0: int, t1: int, device="cpu") -> torch.Tensor:
    """bf16 history slice for all KV heads of request b: [t1 - t0, Hkv, d] (token-major)."""
    return torch.stack([kv_range_bf16(w, which, b, h, t0, t1, device) for h in range(w.Hkv)], 1)


# ----------------------------------------------------------------------------------------------
# NVFP4 encoding of the synthetic data (the stored bytes are the input both sides decode)


def nvfp4_encode(x: torch.Tensor):
    """Encode fp32 rows [..., d] to NVFP4: (codes uint8 [..., d/2], scales uint8 [..., d/16]).

    Scale of each 16-element block: absmax / 6 rounded to E4M3 (nearest-even, clamped to 448).
    Codes: x / scale rounded to the nearest E2M1 value, ties to the even code, saturating at 6.
    Element 2i goes to the low nibble of byte i. A block of zeros gets scale 0 and codes 0.
    """
    *lead, d = x.shape
    assert d % 16 == 0
    xb = x.reshape(*lead, d // 16, 16).to(torch.float32)
    amax = xb.abs().amax(-1)
    s8 = (amax / 6.0).clamp(max=448.0).to(torch.float8_e4m3fn)
    sd = s8.to(torch.float32)
    y = xb / torch.where(sd > 0, sd, torch.ones_like(sd))[..., None]
    a = y.abs()
    code = ((a > 0.25).to(torch.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5)
            + (a >= 3.5) + (a > 5.0)).to(torch.uint8)
    code = code | (((y < 0) & (code > 0)).to(torch.uint8) << 3)
    code = code.reshape(*lead, d // 2, 2)
    packed = (code[..., 0] | (code[..., 1] << 4)).contiguous()
    return packed, s8.view(torch.uint8).reshape(*lead, d // 16).contiguous()


def kv_range_nvfp4(w, which, b, h, t0, t1, device="cpu"):
    return nvfp4_encode(kv_range_f32(w, which, b, h, t0, t1, device))


def append_rows(w: Workload, t0: int, t1: int, device="cpu") -> dict:
    """The arguments of one append call for history positions [t0, t1) of every request:
    bf16 k_new/v_new [B, n, Hkv, d] (GQA), NVFP4 codes and scales (GQA NVFP4) or the latent rows
    k_new [B, n, d] (MLA)."""
    if w.kind == "mla":
        c = torch.stack([kv_range_bf16(w, "c", b, 0, t0, t1, device) for b in range(w.B)])
        return dict(k_new=c.contiguous())
    if w.kv_dtype == "nvfp4":
        out = {}
        for which in ("k", "v"):
            codes = [[None] * w.Hkv for _ in range(w.B)]
            scales = [[None] * w.Hkv for _ in range(w.B)]
            for b in range(w.B):
                for h in range(w.Hkv):
                    codes[b][h], scales[b][h] = kv_range_nvfp4(w, which, b, h, t0, t1, device)
            out[which + "_new"] = torch.stack([torch.stack(c, 1) for c in codes]).contiguous()
            out[which + "_scale"] = torch.stack([torch.stack(c, 1) for c in scales]).contiguous()
        return out
    k = torch.stack([kv_tokens(w, "k", b, t0, t1, device) for b in range(w.B)]).contiguous()
    v = torch.stack([kv_tokens(w, "v", b, t0, t1, device) for b in range(w.B)]).contiguous()
    return dict(k_new=k, v_new=v)


# ----------------------------------------------------------------------------------------------
# paging


def shard_capacity(w: Workload, S_max: int | None = None) -> int:
    """Tokens one shard must be able to hold for histories up to S_max tokens (upper bound)."""
    S_max = w.S if S_max is None else S_max
    if w.layout == "contig":
        return w.contig_chunk
    blocks = -(-S_max // w.rr_block)
    return -(-blocks // w.kvp) * w.rr_block


def page_table(w: Workload, S_max: int | None = None, shuffle: bool = True, device="cpu"):
    """int32 [kvp, B, max_pages]: a synthetic fragmented pool where every (shard, request) gets
    its own pages, in a seeded random order when ``shuffle``. Returns (table, num_pages)."""
    max_pages = -(-shard_capacity(w, S_max) // w.page_tokens)
    n = w.kvp * w.B * max_pages
    if shuffle:
        ids = torch.randperm(n, generator=_gen("cpu", w.seed, _TENSOR_IDS["pages"]))
    else:
        ids = torch.arange(n)
    return ids.to(torch.int32).reshape(w.kvp, w.B, max_pages).to(device), n


# ----------------------------------------------------------------------------------------------
# byte model (algorithmic bytes: what a step must move at minimum)


def kv_read_bytes(num_tokens: int, num_kv_heads: int, d: int, elem_bytes: float,
                  k_and_v: bool = True) -> float:
    """Bytes to read the K (and V) rows of ``num_tokens`` tokens for ``num_kv_heads`` heads."""
    return (2 if k_and_v else 1) * num_tokens * num_kv_heads * d * elem_bytes


def kv_bytes_per_token(w: Workload) -> int:
    """Stored bytes one history token costs, over all KV heads."""
    if w.kind == "mla":
        return w.d * 2  # one latent row; V is its first dv columns, read with it
    if w.kv_dtype == "nvfp4":
        return 2 * w.Hkv * (w.d // 2 + w.d // 16)
    return 2 * w.Hkv * w.d * 2


def partial_bytes(w: Workload, lens) -> int:
    """KV history + q read, O_partial and lse written."""
    return (sum(lens) * kv_bytes_per_token(w) + w.B * w.Hq * w.d * 2
            + w.kvp * w.B * w.Hq * (w.dv + 1) * 4)


def combine_bytes(w: Workload, o_bytes: int = 2) -> int:
    """O_partial and lse read, O (bf16) and lse written."""
    return w.kvp * w.B * w.Hq * (w.dv + 1) * 4 + w.B * w.Hq * (w.dv * o_bytes + 4)


def append_bytes(w: Workload, n_new: int = 1) -> int:
    """New K/V rows read and written."""
    return 2 * w.B * n_new * kv_bytes_per_token(w)


def step_bytes(w: Workload, lens, n_new: int = 1) -> int:
    return append_bytes(w, n_new) + partial_bytes(w, lens) + combine_bytes(w)


def partial_flops(w: Workload, lens) -> float:
    """Algorithmic flops of the partial attention: 2 * heads * tokens * (K width + V width)."""
    return 2.0 * w.Hq * sum(lens) * (w.d + w.dv)
