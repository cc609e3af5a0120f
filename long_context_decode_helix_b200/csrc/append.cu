// append.cu -- place new K/V tokens into the sharded, paged pool.
//
// Placement (paper summary "Helix Parallelism ...", fdeinterviews.com, paragraph on the Helix
// layouts; NVIDIA technical blog, Korean edition, KV-cache section, round-robin example): global
// position t of a request lies in block j = t / rr_block, which goes to KVP shard j % kvp; inside the
// shard the token keeps its global order, at local index (j / kvp) * rr_block + t % rr_block. The
// contiguous layout puts t on shard t / contig_chunk at local index t % contig_chunk. Local index l
// lives on the shard's page page_table[s][b][l / page_tokens], slot l % page_tokens.
//
// The copy is bit-exact (16/8/4-byte vector moves). Lengths advance after every copy of the call has
// read the old seq_lens: in the same block when one block holds all of a request's new tokens,
// otherwise in a second one-block kernel on the same stream.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_common.cuh"
#include "internal.h"

namespace helix {
namespace {

constexpr int kAppendThreads = 256;
constexpr int kTokensPerBlock = 64;

struct Placement {
  int shard, local;
};

__device__ __forceinline__ Placement place(long long t, const AppendParams& p) {
  Placement r;
  if (p.layout == HELIX_LAYOUT_RR) {
    const long long j = t / p.rr_block;
    r.shard = (int)(j % p.kvp);
    r.local = (int)((j / p.kvp) * p.rr_block + t % p.rr_block);
  } else {
    r.shard = (int)(t / p.contig_chunk);
    r.local = (int)(t % p.contig_chunk);
  }
  return r;
}

// Tokens of [0, S) that the layout puts on shard s.
__device__ __forceinline__ long long count_on_shard(long long S, int s, const AppendParams& p) {
  if (p.layout == HELIX_LAYOUT_RR) {
    const long long full = S / p.rr_block, rem = S % p.rr_block;
    long long n = (full / p.kvp) * p.rr_block;
    const long long left = full % p.kvp;
    if (s < left) n += p.rr_block;
    if (s == left) n += rem;
    return n;
  }
  const long long lo = (long long)s * p.contig_chunk;
  long long n = S - lo;
  if (n < 0) n = 0;
  if (n > p.contig_chunk) n = p.contig_chunk;
  return n;
}

template <int VEC>
__device__ __forceinline__ void copy_row(uint8_t* dst, const uint8_t* src, int bytes, int lane0,
                                         int nlanes) {
  using T = typename std::conditional<VEC == 16, uint4,
                                      typename std::conditional<VEC == 8, uint2, uint32_t>::type>::type;
  for (int o = lane0 * VEC; o < bytes; o += nlanes * VEC)
    *reinterpret_cast<T*>(dst + o) = *reinterpret_cast<const T*>(src + o);
}

__device__ void copy_bytes(uint8_t* dst, const uint8_t* src, int bytes, int lane0, int nlanes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | bytes;
  if ((a & 15) == 0) copy_row<16>(dst, src, bytes, lane0, nlanes);
  else if ((a & 7) == 0) copy_row<8>(dst, src, bytes, lane0, nlanes);
  else copy_row<4>(dst, src, bytes, lane0, nlanes);
}

// ---- on-device NVFP4 encoding of one bf16 row of 128 elements (one warp; lane l holds elements
// 4l .. 4l+3, so lanes 4k .. 4k+3 hold scale block k). Every rounding decision is taken in fp32:
// scale = E4M3(fp32(absmax / 6)) rounded to nearest even and clamped to 448 (satfinite);
// code = E2M1(fp32(x / scale)) rounded to nearest even, saturating at 6 (x itself when the scale is
// 0); a code whose magnitude rounds to zero is stored as +0.
struct Nvfp4Lane {
  uint32_t codes16;  // 4 codes, element 4l + e in bits [4e, 4e + 4)
  uint32_t scale;    // E4M3 byte of this lane's block
};

__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float r) {
  uint16_t v;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(v) : "f"(0.f), "f"(r));
  return v & 0xFFu;  // the second source lands in the low byte
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)byte));
  return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}
// two codes in one byte: lo in bits 0-3, hi in bits 4-7
__device__ __forceinline__ uint32_t e2m1x2_rn_satfinite(float lo, float hi) {
  uint16_t v;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u16.u8 %0, t;\n}"
      : "=h"(v) : "f"(hi), "f"(lo));
  uint32_t b = v & 0xFFu;
  if ((b & 0x07u) == 0) b &= 0xF0u;  // -0 -> +0
  if ((b & 0x70u) == 0) b &= 0x0Fu;
  return b;
}

__device__ __forceinline__ Nvfp4Lane encode_lane(const uint8_t* row_bf16, int lane) {
  const uint2 raw = *reinterpret_cast<const uint2*>(row_bf16 + 8 * lane);
  const float x0 = __uint_as_float(raw.x << 16), x1 = __uint_as_float(raw.x & 0xFFFF0000u);
  const float x2 = __uint_as_float(raw.y << 16), x3 = __uint_as_float(raw.y & 0xFFFF0000u);
  float a = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  Nvfp4Lane r;
  r.scale = e4m3_rn_satfinite(__fdiv_rn(a, 6.f));
  const float sd = e4m3_to_f32(r.scale);
  float y0 = x0, y1 = x1, y2 = x2, y3 = x3;
  if (sd > 0.f) {
    y0 = __fdiv_rn(x0, sd);
    y1 = __fdiv_rn(x1, sd);
    y2 = __fdiv_rn(x2, sd);
    y3 = __fdiv_rn(x3, sd);
  }
  r.codes16 = e2m1x2_rn_satfinite(y0, y1) | (e2m1x2_rn_satfinite(y2, y3) << 8);
  return r;
}

__device__ __forceinline__ int rows_of(const AppendParams& p, int b) {
  if (p.n_valid == nullptr) return p.n_new;
  return min(max(p.n_valid[b], 0), p.n_new);
}

__device__ void update_lengths(const AppendParams& p, int b) {
  const int rows = rows_of(p, b);
  if (rows == 0) return;  // leave the lengths of requests without new rows untouched
  const long long S_old = p.seq_lens[b];
  const long long S_new = S_old + rows;
  for (int s = 0; s < p.kvp; ++s) {
    const long long add = count_on_shard(S_new, s, p) - count_on_shard(S_old, s, p);
    p.shard_lens[s * p.B + b] += (int)add;
  }
  p.seq_lens[b] = (int)S_new;
}

// grid: (token blocks, B). One warp copies one (token, head) row set at a time.
__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendParams p,
                                                                bool update_here) {
  const int b = blockIdx.y;
  const long long S_old = p.seq_lens[b];
  const int j0 = blockIdx.x * kTokensPerBlock;
  const int j1 = min(rows_of(p, b), j0 + kTokensPerBlock);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kAppendThreads / 32;
  const int items = max(j1 - j0, 0) * p.Hkv;
  for (int it = warp; it < items; it += nwarps) {
    const int j = j0 + it / p.Hkv;
    const int h = it % p.Hkv;
    const long long t = S_old + j;
    const Placement pl = place(t, p);
    if (pl.shard >= p.kvp) {
      if (lane == 0) raise_dev_error(p.err, HELIX_DEVERR_SHARD);
      continue;
    }
    const int pi = pl.local / p.page_tokens;
    const int slot = pl.local % p.page_tokens;
    if (pi >= p.max_pages) {
      if (lane == 0) raise_dev_error(p.err, HELIX_DEVERR_CAPACITY);
      continue;
    }
    const int page = p.page_table[((size_t)pl.shard * p.B + b) * p.max_pages + pi];
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) raise_dev_error(p.err, HELIX_DEVERR_PAGE_ID);
      continue;
    }
    const size_t src_row = ((size_t)b * p.n_new + j) * p.Hkv + h;
    const size_t dst_row = ((size_t)page * p.Hkv + h) * p.page_tokens + slot;
    if (p.quantize) {
      // d = 128: K codes row of 64 bytes (lane l: bytes 2l, 2l+1), 8 scale bytes, V codes into the
      // token-pair layout (lane l: column word l), V scales block-major
      const Nvfp4Lane k = encode_lane(p.src[0] + src_row * 256, lane);
      const Nvfp4Lane v = encode_lane(p.src[1] + src_row * 256, lane);
      *reinterpret_cast<uint16_t*>(p.dst[0] + dst_row * 64 + 2 * lane) = (uint16_t)k.codes16;
      if ((lane & 3) == 0) p.dst[2][dst_row * 8 + (lane >> 2)] = (uint8_t)k.scale;
      const int pair = slot / 2, shift = 4 * (slot & 1);
      uint32_t* vblk = reinterpret_cast<uint32_t*>(
          p.dst[1] + (((size_t)page * p.Hkv + h) * (p.page_tokens / 2) + pair) * 128);
      uint32_t bits = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) bits |= ((v.codes16 >> (4 * e)) & 0xFu) << (8 * e + shift);
      const int wd = lane;  // columns 4 wd .. 4 wd + 3
      const int sw = ((((wd >> 2) ^ ((pair & 3) << 1))) << 2) | (wd & 3);
      atomicAnd(vblk + sw, ~(0x0F0F0F0Fu << shift));
      atomicOr(vblk + sw, bits);
      if ((lane & 3) == 0)
        p.dst[3][(((size_t)page * p.Hkv + h) * 8 + (lane >> 2)) * p.page_tokens + slot] =
            (uint8_t)v.scale;
    } else if (!p.v_nvfp4) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rb = p.row_bytes[k];
        if (rb == 0) continue;
        copy_bytes(p.dst[k] + dst_row * rb, p.src[k] + src_row * rb, rb, lane, 32);
      }
    } else {
      // K codes and scales: natural rows
      copy_bytes(p.dst[0] + dst_row * p.row_bytes[0], p.src[0] + src_row * p.row_bytes[0],
                 p.row_bytes[0], lane, 32);
      copy_bytes(p.dst[2] + dst_row * p.row_bytes[2], p.src[2] + src_row * p.row_bytes[2],
                 p.row_bytes[2], lane, 32);
      // V codes: element c of this token goes to nibble (slot & 1) of byte [slot / 2][c] of the
      // (page, head) block, whose 16-byte chunks are XOR-swizzled by 2 (pair mod 4) (see helix.h).
      // The other nibble belongs to the neighbouring token, which another warp (or another call)
      // may be writing, so each 32-bit word is updated with atomic and/or.
      const int d = p.row_bytes[1] * 2;
      const int pair = slot / 2;
      const uint8_t* vs = p.src[1] + src_row * p.row_bytes[1];
      uint32_t* vblk = reinterpret_cast<uint32_t*>(
          p.dst[1] + (((size_t)page * p.Hkv + h) * (p.page_tokens / 2) + pair) * d);
      const int shift = 4 * (slot & 1);
      for (int wd = lane; wd < d / 4; wd += 32) {  // word wd covers columns 4wd .. 4wd+3
        const uint32_t two = *reinterpret_cast<const uint16_t*>(vs + 2 * wd);  // 4 codes
        uint32_t bits = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) bits |= ((two >> (4 * e)) & 0xFu) << (8 * e + shift);
        const int sw = ((((wd >> 2) ^ ((pair & 3) << 1))) << 2) | (wd & 3);
        atomicAnd(vblk + sw, ~(0x0F0F0F0Fu << shift));
        atomicOr(vblk + sw, bits);
      }
      // V scales: block-major, [block][token] inside the (page, head) block
      const int nblk = p.row_bytes[3];
      const uint8_t* ss = p.src[3] + src_row * nblk;
      uint8_t* sblk = p.dst[3] + ((size_t)page * p.Hkv + h) * nblk * p.page_tokens;
      for (int k = lane; k < nblk; k += 32) sblk[(size_t)k * p.page_tokens + slot] = ss[k];
    }
  }
  if (update_here) {
    __syncthreads();
    if (threadIdx.x == 0) update_lengths(p, b);
  }
}

__global__ void append_lengths_kernel(const AppendParams p) {
  for (int b = threadIdx.x; b < p.B; b += blockDim.x) update_lengths(p, b);
}

}  // namespace

helix_status append_launch(const AppendParams& p, cudaStream_t stream) {
  if (p.n_new == 0) return HELIX_OK;
  const int nblk = (p.n_new + kTokensPerBlock - 1) / kTokensPerBlock;
  const bool one_block = nblk == 1;
  append_kernel<<<dim3(nblk, p.B), kAppendThreads, 0, stream>>>(p, one_block);
  if (cudaGetLastError() != cudaSuccess) return HELIX_ERR_CUDA;
  if (!one_block) {
    append_lengths_kernel<<<1, 128, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return HELIX_ERR_CUDA;
  }
  return HELIX_OK;
}

}  // namespace helix
