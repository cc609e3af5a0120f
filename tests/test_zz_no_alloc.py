"""helix_attn_partial_noalloc against helix_attn_partial, through the C ABI.

The no-allocation entry point serves callers that cannot give the library a scratch buffer (for
example a plugin whose host application owns all device memory, or a loop that must never call
cudaMalloc). It must give the same partial outputs as the workspace entry point, call after call,
even though every call reuses the same library-owned scratch array.

This file is named so pytest collects it last.
"""

import ctypes

import pytest
import torch

import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu


def _noalloc(hx, cache, q, scale, o_part, lse):
    return hx.lib.helix_attn_partial_noalloc(
        ctypes.byref(cache.struct), ctypes.c_void_p(q.data_ptr()), q.shape[1],
        ctypes.c_float(scale), ctypes.c_void_p(o_part.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    hx = _gpu.hx()
    # long enough histories that units are split across CTAs: the scratch tickets and segment
    # records are exercised, and a stale ticket from the first call would corrupt the second
    w = wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=32, Hkv=2, S=40000)
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, [40000, 23456], chunk=8192)
    q = wl.query(w, "cuda")
    need = hx.workspace_size(cache, w.Hq)
    assert 0 < need <= 4 << 20  # fits HELIX_NOALLOC_SCRATCH_BYTES
    ref_o, ref_lse = hx.partial(cache, q, w.softmax_scale)
    torch.cuda.synchronize()
    for call in range(2):
        o_part = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _noalloc(hx, cache, q, w.softmax_scale, o_part, lse) == 0
        torch.cuda.synchronize()
        _gpu.assert_close_O(o_part.cpu().numpy(), ref_o.cpu().numpy(), f"O_partial, call {call}")
        _gpu.assert_close_lse(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"lse, call {call}")
    assert cache.err_bits() == 0


def test_noalloc_rejects_bad_arguments_without_launching():
    hx = _gpu.hx()
    w = wl.WORKLOADS["gqa_s128k"].with_(B=1, Hq=16, Hkv=1, S=128)
    cache = _gpu.make_cache(w)
    q = wl.query(w, "cuda")
    o_part = torch.empty(w.kvp, 1, 16, 128, device="cuda")
    lse = torch.empty(w.kvp, 1, 16, device="cuda")
    assert _noalloc(hx, cache, q, w.softmax_scale, o_part, lse) == 0
    q32 = torch.zeros(1, 32, 128, dtype=torch.bfloat16, device="cuda")  # 32 heads per KV head
    assert _noalloc(hx, cache, q32, w.softmax_scale, o_part, lse) == 2  # HELIX_ERR_UNSUPPORTED
    assert _noalloc(hx, cache, q, -1.0, o_part, lse) == 1  # HELIX_ERR_INVALID_ARG
