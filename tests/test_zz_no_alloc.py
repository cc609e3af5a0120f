"""helix_attn_partial_noalloc against helix_attn_partial, through the C ABI.

The no-allocation entry point serves callers that cannot give the library a scratch buffer (for
example a plugin whose host application owns all device memory, or a loop that must never call
cudaMalloc). It runs the same kernels as the workspace entry point, on a library-owned array that
every call shares and zeroes before use, so its outputs must be bit-identical to the workspace
call's, call after call: a ticket or segment record left over from an earlier call would change
them.

This file is named so pytest collects it last.
"""

import ctypes

import pytest
import torch

import workloads as wl
import _gpu

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 48 << 20  # HELIX_NOALLOC_SCRATCH_BYTES


def _noalloc(hx, cache_struct, q, scale, o_part, lse):
    return hx.lib.helix_attn_partial_noalloc(
        ctypes.byref(cache_struct), ctypes.c_void_p(q.data_ptr()), q.shape[1],
        ctypes.c_float(scale), ctypes.c_void_p(o_part.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _mla_many(B, seed):
    import numpy as np

    rng = np.random.default_rng(seed)
    lens = [int(x) for x in rng.integers(1, 131, size=B)]
    return wl.WORKLOADS["mla_s1m"].with_(B=B, S=max(lens), kvp=8), lens


CASES = {
    # long enough histories that units are split across CTAs: the scratch tickets and segment
    # records are used, and a stale ticket from the first call would corrupt the second
    "gqa_bf16": (wl.WORKLOADS["gqa_s128k"].with_(B=2, Hq=32, Hkv=2, S=40000), [40000, 23456]),
    "gqa_nvfp4": (wl.WORKLOADS["gqa_nvfp4_s1m"].with_(B=2, Hq=32, Hkv=2, S=40000), [40000, 23456]),
    "mla_split": (wl.WORKLOADS["mla_s1m"].with_(B=2, S=40000, kvp=2), [40000, 25000]),
    # 240 requests x 8 shards: more units than one launch holds, so consecutive launches share
    # the array (each starts from the tickets the previous one returned to zero)
    "mla_many_launches": _mla_many(240, 11),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_equals_workspace_entry_point_on_two_calls(name):
    hx = _gpu.hx()
    w, lens = CASES[name]
    cache = _gpu.make_cache(w)
    _gpu.fill(cache, w, lens, chunk=8192)
    q = wl.query(w, "cuda")
    need = hx.workspace_size(cache, w.Hq)
    assert 0 < need <= NOALLOC_BYTES
    ref_o, ref_lse = hx.partial(cache, q, w.softmax_scale)
    torch.cuda.synchronize()
    for call in range(2):
        o_part = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert _noalloc(hx, cache.struct, q, w.softmax_scale, o_part, lse) == 0
        torch.cuda.synchronize()
        assert torch.equal(o_part, ref_o), f"{name}: O_partial differs on call {call}"
        assert torch.equal(lse, ref_lse), f"{name}: lse differs on call {call}"
    assert cache.err_bits() == 0


def test_noalloc_rejects_bad_arguments_without_launching():
    hx = _gpu.hx()
    w = wl.WORKLOADS["gqa_s128k"].with_(B=1, Hq=16, Hkv=1, S=128)
    cache = _gpu.make_cache(w)
    q = wl.query(w, "cuda")
    o_part = torch.empty(w.kvp, 1, 16, 128, device="cuda")
    lse = torch.empty(w.kvp, 1, 16, device="cuda")
    assert _noalloc(hx, cache.struct, q, w.softmax_scale, o_part, lse) == 0
    q32 = torch.zeros(1, 32, 128, dtype=torch.bfloat16, device="cuda")  # 32 heads per KV head
    assert _noalloc(hx, cache.struct, q32, w.softmax_scale, o_part, lse) == 2  # UNSUPPORTED
    assert _noalloc(hx, cache.struct, q, -1.0, o_part, lse) == 1  # INVALID_ARG
    torch.cuda.synchronize()


def test_noalloc_rejects_a_shape_beyond_its_array():
    """A cache shape whose scratch exceeds the array is refused with HELIX_ERR_CAPACITY before
    anything is enqueued (here: two million MLA requests, 16 M split-unit tickets). The kernel
    never runs, so the cache's pointers only need to be valid and aligned."""
    hx = _gpu.hx()
    w = wl.WORKLOADS["mla_s1m"].with_(B=1, S=64, kvp=8)
    small = _gpu.make_cache(w)
    big = hx.CacheStruct.from_buffer_copy(small.struct)
    big.batch = 2_000_000
    big.max_pages_per_shard = 1
    need = ctypes.c_size_t(0)
    assert hx.lib.helix_attn_workspace_size(ctypes.byref(big), 128, ctypes.byref(need)) == 0
    assert need.value > NOALLOC_BYTES
    q = torch.zeros(1, 128, 576, dtype=torch.bfloat16, device="cuda")
    o_part = torch.empty(8, 1, 128, 512, device="cuda")
    lse = torch.empty(8, 1, 128, device="cuda")
    assert _noalloc(hx, big, q, w.softmax_scale, o_part, lse) == 3  # HELIX_ERR_CAPACITY
    torch.cuda.synchronize()
