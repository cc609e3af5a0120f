// noalloc.cu -- helix_attn_partial_noalloc: partial attention without a caller workspace.
//
// Who needs it: a caller that cannot hand the library a device buffer for scratch. Examples are a
// plugin whose host application owns every byte of device memory and exposes no allocator, a
// runtime working inside a fixed, pre-reserved memory budget, and a latency-critical loop that must
// not call cudaMalloc (which can block on the device and may fail under fragmentation). Such a
// caller still provides q, O_partial and lse; only the kernel's scratch (split-unit tickets and
// segment records) moves into a fixed array that the library owns.
//
// The scratch is one file-scope __device__ array of HELIX_NOALLOC_SCRATCH_BYTES. Every GPU that
// loads the library holds its own copy until the process exits. All calls on a device share it and
// it keeps the previous call's contents, so each call first zeroes the part it uses
// (cudaMemsetAsync on the caller's stream, no allocation). Two calls whose executions overlap on
// the GPU (different streams without ordering) race on the array; callers must order them.
//
// Host code cannot use the array's name as a device address: in host code it names a host-side
// stand-in. The device address is looked up with cudaGetSymbolAddress once per device, with that
// device current, on the first call made on it; that first call should therefore be made before
// any stream capture begins. The cached address belongs to the device's context as it was at that
// first call: after cudaDeviceReset on a device this entry point must not be used there again in
// the same process (the library's module, and with it the array, is reloaded at a new address).
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "helix.h"
#include "internal.h"

static __device__ __align__(256) unsigned char helix_noalloc_scratch[HELIX_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (looked up once per device).
helix_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HELIX_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HELIX_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, helix_noalloc_scratch) != cudaSuccess || p == nullptr)
      return HELIX_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HELIX_OK;
}

}  // namespace

extern "C" helix_status helix_attn_partial_noalloc(const helix_kv_cache* cache, const void* q,
                                                   int32_t num_q_heads, float softmax_scale,
                                                   float* o_partial, float* lse,
                                                   helix_stream_t stream) {
  // every argument is checked before anything is enqueued: a rejected call touches neither the
  // stream nor the shared scratch (which an earlier call may still be using)
  size_t need = 0;
  helix_status st = helix::validate_partial_call(cache, q, num_q_heads, softmax_scale, o_partial,
                                                 lse, &need);
  if (st != HELIX_OK) return st;
  if (need > (size_t)HELIX_NOALLOC_SCRATCH_BYTES) return HELIX_ERR_CAPACITY;
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != HELIX_OK) return st;
  if (cudaMemsetAsync(scratch, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HELIX_ERR_CUDA;
  return helix_attn_partial(cache, q, num_q_heads, softmax_scale, o_partial, lse, scratch, need,
                            stream);
}
