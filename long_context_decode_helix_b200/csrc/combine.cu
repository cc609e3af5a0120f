// combine.cu -- exact LSE-rescaling merge of the per-shard partial outputs.
//
// Paper review (jaehun.me), "Prompt 1.3.2 -- The Secret Weapon", boxed equation: the full output is
// the e^{lse_s}-weighted average of the shard outputs. With normalised shard outputs and the largest
// lse factored out, for every (request, query head):
//     M = max_s lse_s,   w_s = exp(lse_s - M),   LSE = M + ln sum_s w_s,   O = sum_s w_s O_s / sum_s w_s
// Shards with lse = -inf get w_s = 0; if every shard is empty, O = 0 and LSE = -inf.
// One warp per (b, h): lanes stride the v_dim columns with float4 loads.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

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
  const int lane = threadIdx.x & 31;
  if (wl >= nrows) return;
  const int warp = row0 + wl;  // (b, h) row of this warp; rows = B * Hq is the shard stride
  float M = -INFINITY;
  for (int s = 0; s < kvp; ++s) M = fmaxf(M, __ldg(lse + (size_t)s * rows + warp));
  const float Mu = M == -INFINITY ? 0.f : M;
  float den = 0.f;
  for (int s = 0; s < kvp; ++s) den += expf(__ldg(lse + (size_t)s * rows + warp) - Mu);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int c = lane * 4; c < v_dim; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < kvp; ++s) {
      const float w = expf(__ldg(lse + (size_t)s * rows + warp) - Mu);
      if (w == 0.f) continue;  // empty shard: its O_s is never read
      const float4 v =
          __ldg(reinterpret_cast<const float4*>(o_part + ((size_t)s * rows + warp) * v_dim + c));
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    if (BF16_OUT) {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(o_out) + (size_t)warp * v_dim + c;
      uint2 packed;
      packed.x = pack_bf16x2(acc.x, acc.y);
      packed.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(o) = packed;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(o_out) + (size_t)warp * v_dim + c) = acc;
    }
  }
  if (lse_out != nullptr && lane == 0)
    lse_out[warp] = den > 0.f ? Mu + logf(den) : -INFINITY;
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
