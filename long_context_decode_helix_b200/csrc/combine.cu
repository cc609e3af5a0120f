// combine.cu -- exact LSE-rescaling merge of the per-shard partial outputs (the formula is in
// combine_row.cuh). One warp per (b, h): lanes stride the v_dim columns with float4 loads.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "combine_row.cuh"
#include "device_common.cuh"
#include "internal.h"

namespace helix {
namespace {

constexpr int kCombineThreads = 256;

template <bool BF16_OUT>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(int kvp, int rows, int row0, int nrows, int v_dim,
                   const float* __restrict__ o_part, const float* __restrict__ lse,
                   void* __restrict__ o_out, float* __restrict__ lse_out) {
  const int wl = (blockIdx.x * kCombineThreads + threadIdx.x) >> 5;
  if (wl >= nrows) return;
  // (b, h) row of this warp; rows = B * Hq is the shard stride
  combine_row<BF16_OUT>(kvp, rows, row0 + wl, v_dim, o_part, lse, o_out, lse_out,
                        threadIdx.x & 31);
}

}  // namespace

helix_status combine_launch(int kvp, int rows, int row0, int nrows, int v_dim,
                            const float* o_partial, const float* lse, void* o_out, int o_dtype,
                            float* lse_out, cudaStream_t stream) {
  if (nrows == 0) return HELIX_OK;
  const int blocks = (nrows * 32 + kCombineThreads - 1) / kCombineThreads;
  if (o_dtype == 0)
    combine_kernel<true><<<blocks, kCombineThreads, 0, stream>>>(kvp, rows, row0, nrows, v_dim,
                                                                 o_partial, lse, o_out, lse_out);
  else
    combine_kernel<false><<<blocks, kCombineThreads, 0, stream>>>(kvp, rows, row0, nrows, v_dim,
                                                                  o_partial, lse, o_out, lse_out);
  return cudaGetLastError() == cudaSuccess ? HELIX_OK : HELIX_ERR_CUDA;
}

}  // namespace helix
