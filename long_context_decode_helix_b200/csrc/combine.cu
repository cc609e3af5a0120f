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

// Combine over separate source buffers (one [B][Hq][v_dim] O array and one [B][Hq] lse array per
// source shard), for the heads [h0, h0 + nh) of every request; one warp per output row.
template <bool BF16_OUT>
__global__ void __launch_bounds__(kCombineThreads)
    combine_sources_kernel(const CombineSources src, int Hq, int h0, int nh, int nrows, int v_dim,
                           void* __restrict__ o_out, float* __restrict__ lse_out) {
  const int wl = (blockIdx.x * kCombineThreads + threadIdx.x) >> 5;
  if (wl >= nrows) return;
  const int b = wl / nh, hh = wl % nh;
  const size_t row = (size_t)b * Hq + h0 + hh;  // row in every source's [B][Hq] layout
  void* o_row = BF16_OUT ? static_cast<void*>(reinterpret_cast<__nv_bfloat16*>(o_out) +
                                              (size_t)wl * v_dim)
                         : static_cast<void*>(reinterpret_cast<float*>(o_out) + (size_t)wl * v_dim);
  combine_row_sources<BF16_OUT>(
      src.n, v_dim, [&](int s) { return __ldcg(src.lse[s] + row); },
      [&](int s) { return src.o[s] + row * v_dim; }, o_row,
      lse_out != nullptr ? lse_out + wl : nullptr, threadIdx.x & 31);
}

}  // namespace

helix_status combine_sources_launch(const CombineSources& src, int B, int Hq, int h0, int nh,
                                    int v_dim, void* o_out, int o_dtype, float* lse_out,
                                    cudaStream_t stream) {
  const int nrows = B * nh;
  if (nrows == 0) return HELIX_OK;
  const int blocks = (nrows * 32 + kCombineThreads - 1) / kCombineThreads;
  if (o_dtype == 0)
    combine_sources_kernel<true><<<blocks, kCombineThreads, 0, stream>>>(src, Hq, h0, nh, nrows,
                                                                         v_dim, o_out, lse_out);
  else
    combine_sources_kernel<false><<<blocks, kCombineThreads, 0, stream>>>(src, Hq, h0, nh, nrows,
                                                                          v_dim, o_out, lse_out);
  return cudaGetLastError() == cudaSuccess ? HELIX_OK : HELIX_ERR_CUDA;
}

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
