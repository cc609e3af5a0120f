// combine_row.cuh -- the LSE-rescaling merge of one (request, head) row over the KVP shards, done
// by one warp. Shared by the combine kernel and the GQA partial kernels' fused combine, so both
// produce bit-identical results.
//
// Paper review (jaehun.me), "Prompt 1.3.2 -- The Secret Weapon", boxed equation, read for
// partials normalised per shard:
//     M = max_s lse_s,   w_s = exp(lse_s - M),   LSE = M + ln sum_s w_s,   O = sum_s w_s O_s / sum_s w_s
// Shards with lse = -inf get w_s = 0 and their O_s is never read; if every shard is empty, O = 0
// and LSE = -inf. Loads go through L2 (ld.cg), so a row written by another CTA of the same launch
// is read correctly once that CTA's writes were fenced and counted.
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "device_common.cuh"
#include "internal.h"

namespace helix {

// The merge of one row over nsrc sources: lse_at(s) is source s's lse of the row, orow_at(s) its O
// row (v_dim floats); lanes stride v_dim by float4. Every caller goes through this one function,
// so the combine kernel, the fused combine and the combine over separate source buffers give
// bit-identical results for the same partials.
template <bool BF16_OUT, class LseAt, class ORowAt>
__device__ __forceinline__ void combine_row_sources(int nsrc, int v_dim, LseAt lse_at,
                                                    ORowAt orow_at, void* o_out_row,
                                                    float* lse_out_elem, int lane) {
  float M = -INFINITY;
  for (int s = 0; s < nsrc; ++s) M = fmaxf(M, lse_at(s));
  const float Mu = M == -INFINITY ? 0.f : M;
  float den = 0.f;
  for (int s = 0; s < nsrc; ++s) den += expf(lse_at(s) - Mu);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int c = lane * 4; c < v_dim; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < nsrc; ++s) {
      const float w = expf(lse_at(s) - Mu);
      if (w == 0.f) continue;  // empty shard: its O_s is never read
      const float4 v = __ldcg(reinterpret_cast<const float4*>(orow_at(s) + c));
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
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(o_out_row) + c;
      uint2 packed;
      packed.x = pack_bf16x2(acc.x, acc.y);
      packed.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(o) = packed;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(o_out_row) + c) = acc;
    }
  }
  if (lse_out_elem != nullptr && lane == 0) *lse_out_elem = den > 0.f ? Mu + logf(den) : -INFINITY;
}

// rows = B * Hq (the shard stride of o_part / lse); row = b * Hq + h; the kvp shards are one
// contiguous [kvp][rows] (lse) and [kvp][rows][v_dim] (O) array
template <bool BF16_OUT>
__device__ __forceinline__ void combine_row(int kvp, int rows, int row, int v_dim,
                                            const float* o_part, const float* lse, void* o_out,
                                            float* lse_out, int lane) {
  void* o_row = BF16_OUT ? static_cast<void*>(reinterpret_cast<__nv_bfloat16*>(o_out) +
                                              (size_t)row * v_dim)
                         : static_cast<void*>(reinterpret_cast<float*>(o_out) +
                                              (size_t)row * v_dim);
  combine_row_sources<BF16_OUT>(
      kvp, v_dim, [&](int s) { return __ldcg(lse + (size_t)s * rows + row); },
      [&](int s) { return o_part + ((size_t)s * rows + row) * v_dim; }, o_row,
      lse_out != nullptr ? lse_out + row : nullptr, lane);
}

// Fused combine of the GQA partial kernels: called by every thread that `sync` covers after the
// CTA has written one unit (b, k, s) of GQA group bk = b * Hkv + k to O_partial / lse. The CTA that
// finishes the last of the group's kvp units merges the group's G rows (one warp per row).
// The merge itself is kept out of line: it runs once per group and must not add to the register
// pressure of the kernels' streaming loops.
static __device__ __noinline__ void combine_group_rows(const GqaParams& p, int bk, int warp,
                                                       int lane, int nwarps) {
  const int b = bk / p.Hkv, k = bk % p.Hkv;
  const int rows = p.B * p.Hq;
  for (int r = warp; r < p.G; r += nwarps) {
    const int row = b * p.Hq + k * p.G + r;
    if (p.o_dtype == 0)
      combine_row<true>(p.kvp, rows, row, p.D, p.o_part, p.lse, p.o_out, p.lse_out, lane);
    else
      combine_row<false>(p.kvp, rows, row, p.D, p.o_part, p.lse, p.o_out, p.lse_out, lane);
  }
}

template <class Sync>
__device__ __forceinline__ void fused_group_combine(const GqaParams& p, int bk, int* flag, Sync sync,
                                                    int tid, int warp, int lane, int nwarps) {
  __threadfence();  // this thread's O_partial / lse writes reach L2 before the count
  sync();
  if (tid == 0) *flag = atomicAdd(&p.gtickets[bk], 1) == p.kvp - 1;
  sync();
  if (*flag) {
    __threadfence();
    combine_group_rows(p, bk, warp, lane, nwarps);
    if (tid == 0) p.gtickets[bk] = 0;  // ready for the next launch
  }
  sync();  // *flag is reused by the next call
}

}  // namespace helix
