"""Python binding of libhelix.so: KV-parallel (sequence-sharded) decode attention on B200.

This module only marshals arguments: it passes torch tensors' device pointers and the current CUDA
stream to the C ABI declared in ``include/helix.h``. Every step of the computation runs in the
library's CUDA kernels. There is no CPU fallback: if ``libhelix.so`` is missing or cannot be loaded,
importing this package raises.

PyTorch is used for device memory and streams only. ``KVCache`` allocates the paged pool and its
bookkeeping tensors with torch and describes them to the library.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhelix.so")

HELIX_OK = 0
STATUS_NAMES = {0: "HELIX_OK", 1: "HELIX_ERR_INVALID_ARG", 2: "HELIX_ERR_UNSUPPORTED",
                3: "HELIX_ERR_CAPACITY", 4: "HELIX_ERR_CUDA", 5: "HELIX_ERR_TIMEOUT"}
DEVERR_PAGE_ID, DEVERR_CAPACITY, DEVERR_SHARD, DEVERR_WAIT_TIMEOUT = 0x1, 0x2, 0x4, 0x8
KV_BF16, KV_NVFP4 = 0, 1
ATTN_GQA, ATTN_MLA = 0, 1
LAYOUT_RR, LAYOUT_CONTIG = 0, 1


class HelixError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class CacheStruct(ctypes.Structure):
    """Mirror of ``helix_kv_cache`` in include/helix.h."""

    _fields_ = [(n, ctypes.c_int32) for n in (
        "kind", "kv_dtype", "layout", "kvp", "batch", "num_kv_heads", "head_dim", "v_dim",
        "page_tokens", "rr_block", "contig_chunk", "num_pages", "max_pages_per_shard", "reserved_")] + [
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("shard_lens", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("err_word", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m long_context_decode_helix_b200._build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    cache_p = ctypes.POINTER(CacheStruct)
    lib.helix_kv_append.argtypes = [cache_p, P, P, P, P, I32, P, P]
    lib.helix_kv_append.restype = I32
    lib.helix_kv_append_quantize.argtypes = [cache_p, P, P, I32, P, P]
    lib.helix_kv_append_quantize.restype = I32
    lib.helix_attn_workspace_size.argtypes = [cache_p, I32, ctypes.POINTER(SZ)]
    lib.helix_attn_workspace_size.restype = I32
    lib.helix_attn_partial.argtypes = [cache_p, P, I32, F32, P, P, P, SZ, P]
    lib.helix_attn_partial.restype = I32
    lib.helix_attn_partial_noalloc.argtypes = [cache_p, P, I32, F32, P, P, P]
    lib.helix_attn_partial_noalloc.restype = I32
    lib.helix_attn_combine.argtypes = [I32, I32, I32, I32, P, P, P, I32, P, P]
    lib.helix_attn_combine.restype = I32
    lib.helix_attn_partial_combine.argtypes = [cache_p, P, I32, F32, P, P, P, I32, P, P, SZ, P]
    lib.helix_attn_partial_combine.restype = I32
    lib.helix_attn_partial_range.argtypes = [cache_p, P, I32, F32, I32, I32, P, P, P, SZ, P]
    lib.helix_attn_partial_range.restype = I32
    lib.helix_attn_combine_range.argtypes = [I32, I32, I32, I32, I32, I32, P, P, P, I32, P, P]
    lib.helix_attn_combine_range.restype = I32
    lib.helix_attn_combine_sources.argtypes = [I32, P, P, I32, I32, I32, I32, I32, P, I32, P, P]
    lib.helix_attn_combine_sources.restype = I32
    lib.helix_attn_overlapped.argtypes = [cache_p, P, I32, F32, I32, P, P, P, I32, P, P, SZ, P, P,
                                          ctypes.POINTER(P)]
    lib.helix_attn_overlapped.restype = I32
    lib.helix_decode_overlapped.argtypes = [cache_p, P, I32, F32, I32, P, P, P, P, I32, P, P, P, P,
                                            I32, P, P, SZ, P, P, ctypes.POINTER(P)]
    lib.helix_decode_overlapped.restype = I32
    lib.helix_stream_wait.argtypes = [P, P, ctypes.c_uint64]
    lib.helix_stream_wait.restype = I32
    lib.helix_status_string.argtypes = [I32]
    lib.helix_status_string.restype = ctypes.c_char_p
    lib.helix_version.argtypes = []
    lib.helix_version.restype = I32
    return lib


lib = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != HELIX_OK:
        raise HelixError(status, what)


@dataclass
class KVCache:
    """A paged, sequence-sharded KV pool for one attention layer, allocated with torch.

    ``page_table`` (int32 [kvp, batch, max_pages_per_shard]) maps each shard's local pages to pool
    pages; by default every (shard, request) gets its own consecutive pages.
    """

    kind: int
    kv_dtype: int
    layout: int
    kvp: int
    batch: int
    num_kv_heads: int
    head_dim: int
    v_dim: int
    max_pages_per_shard: int
    page_tokens: int = 64
    rr_block: int = 16
    contig_chunk: int = 0
    page_table: torch.Tensor | None = None
    num_pages: int | None = None
    device: str | torch.device = "cuda"
    tensors: dict = field(default_factory=dict)

    def __post_init__(self):
        dev = torch.device(self.device)
        if self.page_table is None:
            n = self.kvp * self.batch * self.max_pages_per_shard
            self.page_table = torch.arange(n, dtype=torch.int32).reshape(
                self.kvp, self.batch, self.max_pages_per_shard)
        self.page_table = self.page_table.to(dev, torch.int32).contiguous()
        if self.num_pages is None:
            self.num_pages = int(self.page_table.max().item()) + 1
        P, H, T, d = self.num_pages, self.num_kv_heads, self.page_tokens, self.head_dim
        t = self.tensors
        if self.kind == ATTN_MLA:
            t["k_pool"] = torch.zeros(P, T, d, dtype=torch.bfloat16, device=dev)
        elif self.kv_dtype == KV_NVFP4:  # V is stored token-pair interleaved (see helix.h)
            t["k_pool"] = torch.zeros(P, H, T, d // 2, dtype=torch.uint8, device=dev)
            t["k_scale"] = torch.zeros(P, H, T, d // 16, dtype=torch.uint8, device=dev)
            t["v_pool"] = torch.zeros(P, H, T // 2, d, dtype=torch.uint8, device=dev)
            t["v_scale"] = torch.zeros(P, H, d // 16, T, dtype=torch.uint8, device=dev)
        else:
            for n in ("k_pool", "v_pool"):
                t[n] = torch.zeros(P, H, T, d, dtype=torch.bfloat16, device=dev)
        t["shard_lens"] = torch.zeros(self.kvp, self.batch, dtype=torch.int32, device=dev)
        t["seq_lens"] = torch.zeros(self.batch, dtype=torch.int32, device=dev)
        t["err_word"] = torch.zeros(1, dtype=torch.int32, device=dev)
        self._struct = CacheStruct(
            kind=self.kind, kv_dtype=self.kv_dtype, layout=self.layout, kvp=self.kvp,
            batch=self.batch, num_kv_heads=H, head_dim=d, v_dim=self.v_dim, page_tokens=T,
            rr_block=self.rr_block, contig_chunk=self.contig_chunk, num_pages=P,
            max_pages_per_shard=self.max_pages_per_shard, reserved_=0,
            k_pool=t["k_pool"].data_ptr(),
            v_pool=t["v_pool"].data_ptr() if "v_pool" in t else None,
            k_scale=t["k_scale"].data_ptr() if "k_scale" in t else None,
            v_scale=t["v_scale"].data_ptr() if "v_scale" in t else None,
            page_table=self.page_table.data_ptr(), shard_lens=t["shard_lens"].data_ptr(),
            seq_lens=t["seq_lens"].data_ptr(), err_word=t["err_word"].data_ptr())
        self._workspace = None

    # -- views ------------------------------------------------------------------------------
    @property
    def struct(self) -> CacheStruct:
        return self._struct

    def __getitem__(self, name) -> torch.Tensor:
        return self.tensors[name]

    def err_bits(self) -> int:
        return int(self.tensors["err_word"].item())

    def clear_errors(self):
        self.tensors["err_word"].zero_()

    def workspace(self, num_q_heads: int) -> torch.Tensor:
        """A zero-initialised workspace for ``partial``, kept with the cache and reused."""
        n = workspace_size(self, num_q_heads)
        if self._workspace is None or self._workspace.numel() < n:
            self._workspace = torch.zeros(max(n, 16), dtype=torch.uint8,
                                          device=self.tensors["k_pool"].device)
        return self._workspace


def append(cache: KVCache, k_new, v_new=None, k_scale=None, v_scale=None, n_valid=None,
           stream=None):
    """Append n_new tokens per request (``helix_kv_append``). k_new: [B, n_new, ...].

    ``n_valid`` (device int32 [B], optional): request b appends only its first n_valid[b] rows.
    """
    n_new = int(k_new.shape[1])
    _check(lib.helix_kv_append(ctypes.byref(cache.struct), _ptr(k_new), _ptr(v_new),
                               _ptr(k_scale), _ptr(v_scale), n_new, _ptr(n_valid),
                               _stream(stream)), "helix_kv_append")


def append_quantize(cache: KVCache, k_new, v_new, n_valid=None, stream=None):
    """Append bf16 rows [B, n_new, Hkv, 128] to an NVFP4 cache, encoding them on the device
    (``helix_kv_append_quantize``)."""
    n_new = int(k_new.shape[1])
    _check(lib.helix_kv_append_quantize(ctypes.byref(cache.struct), _ptr(k_new), _ptr(v_new),
                                        n_new, _ptr(n_valid), _stream(stream)),
           "helix_kv_append_quantize")


def workspace_size(cache: KVCache, num_q_heads: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.helix_attn_workspace_size(ctypes.byref(cache.struct), num_q_heads, ctypes.byref(n)),
           "helix_attn_workspace_size")
    return int(n.value)


def partial(cache: KVCache, q: torch.Tensor, softmax_scale: float, o_partial=None, lse=None,
            workspace=None, stream=None):
    """Per-shard partial attention (``helix_attn_partial``): returns (O_partial, lse)."""
    B, Hq, _ = q.shape
    dev = q.device
    if o_partial is None:
        o_partial = torch.empty(cache.kvp, B, Hq, cache.v_dim, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(cache.kvp, B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = cache.workspace(Hq)
    _check(lib.helix_attn_partial(ctypes.byref(cache.struct), _ptr(q), Hq, float(softmax_scale),
                                  _ptr(o_partial), _ptr(lse), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)),
           "helix_attn_partial")
    return o_partial, lse


def combine(o_partial: torch.Tensor, lse: torch.Tensor, out=None, lse_out=None,
            out_dtype=torch.bfloat16, want_lse=True, stream=None):
    """LSE-rescaling combine (``helix_attn_combine``): returns (O, LSE or None)."""
    P, B, Hq, dv = o_partial.shape
    if out is None:
        out = torch.empty(B, Hq, dv, dtype=out_dtype, device=o_partial.device)
    if lse_out is None and want_lse:
        lse_out = torch.empty(B, Hq, dtype=torch.float32, device=o_partial.device)
    o_dtype = 0 if out.dtype == torch.bfloat16 else 1
    _check(lib.helix_attn_combine(P, B, Hq, dv, _ptr(o_partial), _ptr(lse), _ptr(out), o_dtype,
                                  _ptr(lse_out), _stream(stream)), "helix_attn_combine")
    return out, lse_out


MAX_SOURCES = 16


def combine_sources(o_parts, lses, head_begin: int, head_end: int, out=None, lse_out=None,
                    out_dtype=torch.bfloat16, want_lse=True, stream=None, ptrs=None):
    """``helix_attn_combine_sources``: the combine over separate per-shard buffers (O [B][Hq][dv]
    and lse [B][Hq] each) for the heads [head_begin, head_end). ``ptrs`` may give the sources as
    raw device addresses instead (``[(o_addr, lse_addr), ...]``, e.g. other processes' buffers mapped
    into this one); the shapes are then taken from ``o_parts[0]`` / ``lses[0]``. Returns (O, LSE or
    None) with O [B][head_end - head_begin][dv]."""
    B, Hq, dv = o_parts[0].shape
    n = len(ptrs) if ptrs is not None else len(o_parts)
    if ptrs is None:
        if len(lses) != n:
            raise ValueError("one lse buffer per O buffer")
        for o, l in zip(o_parts, lses):
            if tuple(o.shape) != (B, Hq, dv) or tuple(l.shape) != (B, Hq) or not (
                    o.is_contiguous() and l.is_contiguous()):
                raise ValueError("every source is a contiguous O [B][Hq][dv] and lse [B][Hq]")
        ptrs = [(o.data_ptr(), l.data_ptr()) for o, l in zip(o_parts, lses)]
    nh = head_end - head_begin
    dev = o_parts[0].device
    if out is None:
        out = torch.empty(B, nh, dv, dtype=out_dtype, device=dev)
    if lse_out is None and want_lse:
        lse_out = torch.empty(B, nh, dtype=torch.float32, device=dev)
    o_arr = (ctypes.c_void_p * n)(*[o for o, _ in ptrs])
    l_arr = (ctypes.c_void_p * n)(*[l for _, l in ptrs])
    o_dtype = 0 if out.dtype == torch.bfloat16 else 1
    _check(lib.helix_attn_combine_sources(n, o_arr, l_arr, B, Hq, dv, head_begin, head_end,
                                          _ptr(out), o_dtype, _ptr(lse_out), _stream(stream)),
           "helix_attn_combine_sources")
    return out, lse_out


def partial_combine(cache: KVCache, q: torch.Tensor, softmax_scale: float, o_partial=None,
                    lse=None, out=None, lse_out=None, out_dtype=torch.bfloat16, workspace=None,
                    stream=None):
    """Partial attention and the LSE combine in one launch for GQA caches
    (``helix_attn_partial_combine``). Returns (O, LSE)."""
    B, Hq, _ = q.shape
    dev = q.device
    if o_partial is None:
        o_partial = torch.empty(cache.kvp, B, Hq, cache.v_dim, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(cache.kvp, B, Hq, dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty(B, Hq, cache.v_dim, dtype=out_dtype, device=dev)
    if lse_out is None:
        lse_out = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = cache.workspace(Hq)
    o_dtype = 0 if out.dtype == torch.bfloat16 else 1
    _check(lib.helix_attn_partial_combine(ctypes.byref(cache.struct), _ptr(q), Hq,
                                          float(softmax_scale), _ptr(o_partial), _ptr(lse),
                                          _ptr(out), o_dtype, _ptr(lse_out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)), "helix_attn_partial_combine")
    return out, lse_out


def partial_range(cache: KVCache, q: torch.Tensor, softmax_scale: float, b_begin: int, b_end: int,
                  o_partial: torch.Tensor, lse: torch.Tensor, workspace=None, stream=None):
    """``helix_attn_partial_range``: partial attention of requests [b_begin, b_end) only, written
    into the full-shape ``o_partial`` / ``lse``."""
    B, Hq, _ = q.shape
    if workspace is None:
        workspace = cache.workspace(Hq)
    _check(lib.helix_attn_partial_range(ctypes.byref(cache.struct), _ptr(q), Hq,
                                        float(softmax_scale), b_begin, b_end, _ptr(o_partial),
                                        _ptr(lse), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "helix_attn_partial_range")
    return o_partial, lse


def combine_range(o_partial: torch.Tensor, lse: torch.Tensor, b_begin: int, b_end: int, out,
                  lse_out=None, stream=None):
    """``helix_attn_combine_range``: combine of requests [b_begin, b_end) into the full-shape
    ``out`` / ``lse_out``."""
    P, B, Hq, dv = o_partial.shape
    o_dtype = 0 if out.dtype == torch.bfloat16 else 1
    _check(lib.helix_attn_combine_range(P, B, Hq, dv, b_begin, b_end, _ptr(o_partial), _ptr(lse),
                                        _ptr(out), o_dtype, _ptr(lse_out), _stream(stream)),
           "helix_attn_combine_range")
    return out, lse_out


class Overlap:
    """The second stream and the events ``helix_attn_overlapped`` / ``helix_decode_overlapped``
    need, created once (2 * n_groups + 1 events: enough for either call)."""

    def __init__(self, n_groups: int, device=None):
        self.n_groups = int(n_groups)
        self.device = device
        self.stream_b = torch.cuda.Stream(device=device)
        cur = torch.cuda.current_stream(device)
        self.events = [torch.cuda.Event() for _ in range(2 * self.n_groups + 1)]
        for e in self.events:  # torch creates the CUDA event lazily, on its first record
            e.record(cur)
        self._handles = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])
        self._nvalid = {}

    def group_n_valid(self, batch: int, n_new: int, device):
        """int32 [groups][batch]: n_new for the requests of group g in row g, 0 elsewhere."""
        key = (batch, n_new)
        if key not in self._nvalid:
            g = min(self.n_groups, batch)
            per = -(-batch // g)
            t = torch.zeros(g, batch, dtype=torch.int32)
            for i in range(g):
                t[i, i * per:min(batch, (i + 1) * per)] = n_new
            self._nvalid[key] = t.to(device)
        return self._nvalid[key]



def overlapped(cache: KVCache, q: torch.Tensor, softmax_scale: float, overlap: Overlap,
               o_partial=None, lse=None, out=None, lse_out=None, out_dtype=torch.bfloat16,
               workspace=None, stream=None):
    """HOP-B analogue (``helix_attn_overlapped``): per request group, partial attention on
    ``stream`` and the combine on ``overlap.stream_b``, overlapping the next group's partial.
    Returns (O, LSE)."""
    B, Hq, _ = q.shape
    dev = q.device
    if o_partial is None:
        o_partial = torch.empty(cache.kvp, B, Hq, cache.v_dim, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(cache.kvp, B, Hq, dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty(B, Hq, cache.v_dim, dtype=out_dtype, device=dev)
    if lse_out is None:
        lse_out = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = cache.workspace(Hq)
    o_dtype = 0 if out.dtype == torch.bfloat16 else 1
    _check(lib.helix_attn_overlapped(ctypes.byref(cache.struct), _ptr(q), Hq, float(softmax_scale),
                                     overlap.n_groups, _ptr(o_partial), _ptr(lse), _ptr(out),
                                     o_dtype, _ptr(lse_out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(stream), _stream(overlap.stream_b),
                                     overlap._handles), "helix_attn_overlapped")
    return out, lse_out


def decode_overlapped(cache: KVCache, q: torch.Tensor, softmax_scale: float, overlap: Overlap,
                      k_new, v_new=None, k_scale=None, v_scale=None, o_partial=None, lse=None,
                      out=None, lse_out=None, out_dtype=torch.bfloat16, workspace=None,
                      stream=None):
    """HOP-B analogue of a whole decode step (``helix_decode_overlapped``): per request group the
    append and the combine run on ``overlap.stream_b``, overlapping the neighbouring groups'
    partial attention on ``stream``. Returns (O, LSE)."""
    B, Hq, _ = q.shape
    dev = q.device
    n_new = int(k_new.shape[1])
    if o_partial is None:
        o_partial = torch.empty(cache.kvp, B, Hq, cache.v_dim, dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(cache.kvp, B, Hq, dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty(B, Hq, cache.v_dim, dtype=out_dtype, device=dev)
    if lse_out is None:
        lse_out = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = cache.workspace(Hq)
    gnv = overlap.group_n_valid(B, n_new, dev)
    o_dtype = 0 if out.dtype == torch.bfloat16 else 1
    _check(lib.helix_decode_overlapped(ctypes.byref(cache.struct), _ptr(q), Hq,
                                       float(softmax_scale), overlap.n_groups, _ptr(k_new),
                                       _ptr(v_new), _ptr(k_scale), _ptr(v_scale), n_new, _ptr(gnv),
                                       _ptr(o_partial), _ptr(lse), _ptr(out), o_dtype,
                                       _ptr(lse_out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream), _stream(overlap.stream_b),
                                       overlap._handles), "helix_decode_overlapped")
    return out, lse_out


HELIX_ERR_TIMEOUT = 5
_wait_events = {}


def wait(stream=None, limit_s: float = 60.0):
    """Wait for the work enqueued on ``stream`` (default: the current stream) with a wall-clock
    limit (``helix_stream_wait``). Raises ``HelixError`` with status HELIX_ERR_TIMEOUT when the limit
    passes first (the work stays enqueued), HELIX_ERR_CUDA when the stream's work failed."""
    s = torch.cuda.current_stream() if stream is None else stream
    ev = _wait_events.get(s.device)
    if ev is None:
        ev = torch.cuda.Event()
        ev.record(s)  # torch creates the CUDA event lazily, on its first record
        _wait_events[s.device] = ev
    _check(lib.helix_stream_wait(_stream(s), ctypes.c_void_p(ev.cuda_event),
                                 int(max(0.0, limit_s) * 1e6)), "helix_stream_wait")


def decode_step(cache: KVCache, q, k_new, v_new=None, softmax_scale=None, k_scale=None,
                v_scale=None, o_partial=None, lse=None, out=None, lse_out=None, stream=None):
    """One decode-attention layer step: append the new token, then partial attention and the
    combine (one launch for GQA caches, ``helix_attn_partial_combine``). Returns (O, LSE)."""
    if softmax_scale is None:
        softmax_scale = cache.head_dim ** -0.5
    append(cache, k_new, v_new, k_scale, v_scale, stream=stream)
    return partial_combine(cache, q, softmax_scale, o_partial, lse, out, lse_out, stream=stream)
