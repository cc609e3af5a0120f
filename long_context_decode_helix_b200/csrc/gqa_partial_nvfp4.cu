// gqa_partial_nvfp4.cu -- per-shard partial decode attention for grouped-query attention over an
// NVFP4 KV cache (the pages' simulated results read "FP4" KV: paper summary, roofline paragraph).
//
// Same result as the bf16 kernel (paper summary, paragraph on KV parallelism): for every request b,
// KV head k and KVP shard s, over the shard's tokens T_s,
//     z_{h,t} = scale * <q_{b,h}, K_{t,k}>  for the G <= 16 query heads h of KV head k,
//     O_s[h] = sum_t e^{z - m} V_t / sum_t e^{z - m},   lse_s[h] = m + ln sum_t e^{z - m},
// with K and V decoded from E2M1 codes times one E4M3 scale per 16 elements along d. The products
// are exact in f16 (at most 6 significant bits, 2^-10 .. 2688), so the tensor cores see exactly the
// decoded cache.
//
// Why its own kernel: at 4.5 bits per element the cache streams four times faster than bf16, and
// every element has to be decoded in registers (a cvt of two codes and an f16x2 multiply by their
// scale per pair), so the per-token instruction count, not HBM, bounds a kernel that spreads a page
// over four warps. Here one warp owns a whole 64-token page: 8 warps work on 8 different pages,
// every page-level step (row max, rescale decision, shuffles) is amortised over 64 tokens, and the
// eight n-tiles of the page give eight independent MMA chains for S.
//
// Per page and warp (16 head rows = the M of an m16n8k16 tile, f16 in, fp32 accumulate):
//   S = q K^T: a lane reads 16 code bytes (32 elements) of one token per n-tile; the MMA's k index
//     is permuted so those bytes are its B operands for all eight k-steps (q's A fragments use the
//     same permutation).
//   P V: V is stored token-pair interleaved (byte = the codes of tokens 2i and 2i+1 in one column)
//     with its n index permuted (n-tile j holds columns 16 n + j), so one 16-byte load per token
//     pair feeds all sixteen n-tiles; the segment flush writes O in natural column order.
//   Row sums of P come from one extra MMA against a column of ones, so they are the sums of exactly
//     the f16 weights that multiplied V; they normalise O and give the LSE (f16 weights carry a
//     relative error below 2^-11, so the LSE error stays below 5e-4).
//   Softmax is online in fp32 and base 2. The reference maximum moves lazily, only when a row
//     maximum exceeds it by more than 8, so weights stay below 2^8 and O is rarely rescaled.
//
// Work split and merging are those of the bf16 kernel: the (b, k, s) units are laid end to end as
// one list of pages and every persistent CTA takes an equal contiguous range; units cut by range
// boundaries are merged by the last CTA to arrive on the unit's ticket. There is no producer warp
// (eight warps leave each thread up to 255 registers): warp w takes pages w, w + 8, w + 16, ... of
// the range and loads them itself -- four bulk copies (K codes, K scales, V codes, V scales) per page
// into its two ring slots; after finishing a page it refills the slot with its page two ahead, so
// 16 pages per SM are in flight. Page ids are resolved 32 at a time, one per lane, a batch ahead.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "combine_row.cuh"
#include "device_common.cuh"
#include "internal.h"

namespace helix {
namespace {

constexpr int kD = 128;
constexpr int kPage = 64;
constexpr int kRows = 16;
constexpr int kWarps = 8;  // one page each; each owns ring slots 2 w and 2 w + 1
constexpr int kThreads = kWarps * 32;
// the fixed-order merge of the warps' O and the segment flush's (row, column) split of the threads
// are written for exactly this count
static_assert(kWarps == 8 && kThreads == 16 * 16, "segment flush written for eight warps");
constexpr int kNStage = 2 * kWarps;
constexpr int kKcBytes = kPage * kD / 2;   // 4096
constexpr int kKsBytes = kPage * kD / 16;  // 512
constexpr int kOffKs = kKcBytes, kOffVc = kKcBytes + kKsBytes, kOffVs = 2 * kKcBytes + kKsBytes;
constexpr int kStageBytes = 2 * (kKcBytes + kKsBytes);  // 9216
constexpr int kRec = kRows * (kD + 3);                  // workspace record: O, m, (unused), lb
constexpr float kLazy = 8.f;  // base-2 headroom before the reference maximum moves
constexpr int kMinPagesPerCta = 4;
constexpr uint32_t kOnes = 0x3C003C00u;  // f16x2 (1, 1)

struct Tail {
  uint64_t full[kNStage];
  float mstat[kWarps][kRows];
  float lstat[kWarps][kRows];
  int flag;
  int gflag;
};

constexpr size_t smem_fixed() {
  return 1024 + (size_t)kNStage * kStageBytes + 2 * (size_t)kRows * kD * sizeof(float) +
         sizeof(Tail);
}

__device__ __forceinline__ long long range_begin(int c, long long W, int G) {
  return (long long)c * W / G;
}
__device__ __forceinline__ int cta_of(long long x, long long W, int G) {
  return (int)(((x + 1) * (long long)G - 1) / W);
}

__device__ __forceinline__ void e2m1x4_to_f16x2(uint32_t w, uint32_t& h0, uint32_t& h1,
                                                uint32_t& h2, uint32_t& h3) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
}
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  return h;
}
// codes (f16x2) times the low or the high half of a scale pair, broadcast to both halves
__device__ __forceinline__ uint32_t mul_lo(uint32_t codes, uint32_t sc2) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&codes),
                            __low2half2(*reinterpret_cast<const __half2*>(&sc2)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t mul_hi(uint32_t codes, uint32_t sc2) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&codes),
                            __high2half2(*reinterpret_cast<const __half2*>(&sc2)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a),
                            *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// fma(a0, b, c), fma(a1, b, c) in one instruction (two IEEE round-to-nearest fused multiply-adds)
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %4};\n"
      " mov.b64 rc, {%5, %5};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d0), "=f"(d1) : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// max(a, b, c) in one instruction
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16x2(bf16_lo_to_f32(v), bf16_hi_to_f32(v));
}

__global__ void __launch_bounds__(kThreads, 1) gqa_partial_nvfp4_kernel(const GqaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* Obuf = reinterpret_cast<float*>(smem + (size_t)kNStage * kStageBytes);
  Tail* tail = reinterpret_cast<Tail*>(Obuf + 2 * kRows * kD);
  int* pre = reinterpret_cast<int*>(tail + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int U = p.units;

  // ---- per-unit page counts and their prefix sums (every CTA computes the same table) ----
  for (int u = tid; u < U; u += kThreads) {
    const int s = (u + p.u0) % p.kvp;
    const int b = ((u + p.u0) / p.kvp) / p.Hkv;
    const int len = p.shard_lens[s * p.B + b];
    int np = len > 0 ? (len + kPage - 1) / kPage : 0;
    if (np > p.max_pages) {
      if (blockIdx.x == 0) raise_dev_error(p.err, HELIX_DEVERR_CAPACITY);
      np = p.max_pages;
    }
    pre[u + 1] = np;
  }
  if (tid == 0) {
    pre[0] = 0;
    tail->flag = 0;
    for (int i = 0; i < kNStage; ++i) mbar_init(&tail->full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of pre[1..U]
    const int per = (U + 31) / 32;
    const int lo = 1 + lane * per, hi = min(U + 1, lo + per);
    int run = 0;
    for (int i = lo; i < hi; ++i) run += pre[i];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int acc = incl - run;
    for (int i = lo; i < hi; ++i) {
      acc += pre[i];
      pre[i] = acc;
    }
  }
  __syncthreads();

  const long long W = pre[U];
  // units with no tokens: O_s = 0, lse_s = -inf
  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    if (pre[u + 1] != pre[u]) continue;
    const int s = (u + p.u0) % p.kvp, bk = (u + p.u0) / p.kvp, k = bk % p.Hkv, b = bk / p.Hkv;
    const size_t row0 = ((size_t)s * p.B + b) * p.Hq + (size_t)k * p.G;
    for (int i = tid; i < p.G * kD; i += kThreads) p.o_part[row0 * kD + i] = 0.f;
    for (int i = tid; i < p.G; i += kThreads) p.lse[row0 + i] = -INFINITY;
    if (p.o_out != nullptr)
      fused_group_combine(p, bk, &tail->gflag, [] { __syncthreads(); }, tid, warp, lane, kWarps);
  }
  // at least kMinPagesPerCta pages per CTA: short histories would otherwise be cut into one-page
  // pieces whose merges cost more than the pages (measured on the 4K-token workload)
  const int Geff = (int)min((long long)gridDim.x, (W + kMinPagesPerCta - 1) / kMinPagesPerCta);
  if ((int)blockIdx.x >= Geff) return;
  const long long g_begin = range_begin(blockIdx.x, W, Geff);
  const long long g_end = range_begin(blockIdx.x + 1, W, Geff);
  int u_first;
  {
    int lo = 0, hi = U;  // last u with pre[u] <= g_begin
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= g_begin) lo = mid; else hi = mid;
    }
    u_first = lo;
    while (pre[u_first + 1] <= g_begin) ++u_first;
  }

  const int g8 = lane >> 2;  // fragment rows g8 and g8 + 8 (query heads of the group)
  const int t4 = lane & 3;

  // ---- this warp's pages: j-th own page = range page warp + 8 j, ring slot 2 warp + (j & 1) ----
  const long long w_range = g_end - g_begin;
  const int n_own = w_range > warp ? (int)((w_range - warp + kWarps - 1) / kWarps) : 0;
  // pool page-head index (page * Hkv + kv head) of own page 32 jb + lane; -1 = none or a bad id
  auto resolve = [&](int jb) -> int {
    const int jj = 32 * jb + lane;
    if (jj >= n_own) return -1;
    const long long g = g_begin + warp + (long long)kWarps * jj;
    int lo = 0, hi = U;  // the last unit with pre[lo] <= g, which holds page g
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= g) lo = mid; else hi = mid;
    }
    const int s = (lo + p.u0) % p.kvp, bk = (lo + p.u0) / p.kvp;
    const int b = bk / p.Hkv, k = bk % p.Hkv;
    const int page = __ldg(p.page_table + ((size_t)s * p.B + b) * p.max_pages + (int)(g - pre[lo]));
    if (page < 0 || page >= p.num_pages) {
      raise_dev_error(p.err, HELIX_DEVERR_PAGE_ID);
      return -1;
    }
    return page * p.Hkv + k;
  };
  // Starts the loads of own page j (page-head id) into its slot; a page without data completes the
  // slot's phase with a plain arrive, so the phase count stays in step either way.
  auto issue = [&](int j, int id) {
    if (lane == 0) {
      const int slot = 2 * warp + (j & 1);
      if (id < 0) {
        mbar_arrive(&tail->full[slot]);
      } else {
        uint8_t* st = stages + (size_t)slot * kStageBytes;
        const size_t ph = (size_t)id;
        fence_proxy_async_smem();  // this warp's reads of the slot's previous page come first
        mbar_arrive_expect_tx(&tail->full[slot], kStageBytes);
        bulk_load(st, p.k_codes + ph * kKcBytes, kKcBytes, &tail->full[slot]);
        bulk_load(st + kOffKs, p.k_scale + ph * kKsBytes, kKsBytes, &tail->full[slot]);
        bulk_load(st + kOffVc, p.v_codes + ph * kKcBytes, kKcBytes, &tail->full[slot]);
        bulk_load(st + kOffVs, p.v_scale + ph * kKsBytes, kKsBytes, &tail->full[slot]);
      }
    }
  };
  int ids_cur = resolve(0), ids_nxt = resolve(1);  // own pages [32 jb, 32 jb + 64), jb = j / 32
  int issued = 0;                                  // own pages whose loads have been started
  for (; issued < min(2, n_own); ++issued) issue(issued, __shfl_sync(0xffffffffu, ids_cur, issued));

  uint32_t qa[8][4];  // q as f16 A fragments, permuted k (see the header)
  float O[16][4];     // n-tile j holds output columns 16 n + j
  float lb[4];        // P row sums from the ones-column MMA ([0]: row g8, [2]: row g8 + 8)
  float m_ref[2];     // reference maximum per row (base-2 logits)
  auto reset_state = [&]() {
#pragma unroll
    for (int j = 0; j < 16; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
    lb[0] = lb[1] = lb[2] = lb[3] = 0.f;
    m_ref[0] = m_ref[1] = -INFINITY;
  };
  int s_u = 0, b_u = 0, k_u = 0, len_u = 0;
  auto enter_unit = [&](int uu) {
    s_u = (uu + p.u0) % p.kvp;
    const int bk = (uu + p.u0) / p.kvp;
    k_u = bk % p.Hkv;
    b_u = bk / p.Hkv;
    len_u = p.shard_lens[s_u * p.B + b_u];
    const __nv_bfloat16* qb = p.q + ((size_t)b_u * p.Hq + (size_t)k_u * p.G) * kD;
    const bool v0 = g8 < p.G, v1 = g8 + 8 < p.G;
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qb + (size_t)g8 * kD);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(qb + (size_t)(g8 + 8) * kD);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      // logical columns (2t, 2t+1 | 2t+8, 2t+9) of k-step kk are head-dim elements
      // 32t + 4kk + (0, 1 | 2, 3); q is rounded to f16 (exact for 2^-14 <= |q| <= 65504)
      const int c0 = 32 * t4 + 4 * kk;
      qa[kk][0] = v0 ? bf16x2_to_f16x2(__ldg(r0 + c0 / 2)) : 0u;
      qa[kk][1] = v1 ? bf16x2_to_f16x2(__ldg(r1 + c0 / 2)) : 0u;
      qa[kk][2] = v0 ? bf16x2_to_f16x2(__ldg(r0 + c0 / 2 + 1)) : 0u;
      qa[kk][3] = v1 ? bf16x2_to_f16x2(__ldg(r1 + c0 / 2 + 1)) : 0u;
    }
  };

  bool dead = false;
  const float sl2 = p.scale_log2;

  // One page (64 tokens, nvalid of them in the history) from ring stage st, all at once: eight
  // n-tiles of S (eight independent MMA chains), one softmax pass and one rescale decision for the
  // page, then P V over four 16-token k-chunks.
  auto process_page = [&](const uint8_t* st, int nvalid) {
    // ---- S = q K^T: n-tile n holds tokens 8 n + (0..7); this lane's token of n-tile n is 8n + g8
    float s[8][4];
    {
      uint4 kc[8];
      uint32_t sc2[8];  // (scale of elements [32 t, 32 t + 16), of [32 t + 16, 32 t + 32))
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int token = 8 * n + g8;
        kc[n] = *reinterpret_cast<const uint4*>(st + token * (kD / 2) + t4 * 16);
        sc2[n] =
            e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(st + kOffKs + token * 8 + 2 * t4));
        s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
      }
#pragma unroll
      for (int wq = 0; wq < 4; ++wq) {  // code word wq holds k-steps 2 wq and 2 wq + 1
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const uint32_t word = wq == 0 ? kc[n].x : wq == 1 ? kc[n].y : wq == 2 ? kc[n].z : kc[n].w;
          uint32_t h0, h1, h2, h3;
          e2m1x4_to_f16x2(word, h0, h1, h2, h3);
          if (wq < 2) {
            mma_f16_16816(s[n], qa[2 * wq], mul_lo(h0, sc2[n]), mul_lo(h1, sc2[n]));
            mma_f16_16816(s[n], qa[2 * wq + 1], mul_lo(h2, sc2[n]), mul_lo(h3, sc2[n]));
          } else {
            mma_f16_16816(s[n], qa[2 * wq], mul_hi(h0, sc2[n]), mul_hi(h1, sc2[n]));
            mma_f16_16816(s[n], qa[2 * wq + 1], mul_hi(h2, sc2[n]), mul_hi(h3, sc2[n]));
          }
        }
      }
    }
    // ---- online softmax over the page (base 2, lazy reference maximum). The logit scale (times
    // log2 e, positive) is applied inside the exponent, fma(s, sl2, -m); the row maximum is taken
    // over the raw scores and scaled once.
    if (nvalid < kPage) {
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int t = 8 * n + 2 * t4;
        if (t >= nvalid) s[n][0] = s[n][2] = -INFINITY;
        if (t + 1 >= nvalid) s[n][1] = s[n][3] = -INFINITY;
      }
    }
    float mx0 = fmaxf(s[0][0], s[0][1]), mx1 = fmaxf(s[0][2], s[0][3]);
#pragma unroll
    for (int n = 1; n < 8; ++n) {
      mx0 = max3f(mx0, s[n][0], s[n][1]);
      mx1 = max3f(mx1, s[n][2], s[n][3]);
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2)) * sl2;
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2)) * sl2;
    const bool up0 = mx0 > m_ref[0] + kLazy, up1 = mx1 > m_ref[1] + kLazy;
    if (__any_sync(0xffffffffu, up0 || up1)) {
      const float n0 = up0 ? mx0 : m_ref[0], n1 = up1 ? mx1 : m_ref[1];
      const float a0 = up0 ? fast_exp2(m_ref[0] - n0) : 1.f;  // exp2(-inf) = 0 at the start
      const float a1 = up1 ? fast_exp2(m_ref[1] - n1) : 1.f;
      m_ref[0] = n0;
      m_ref[1] = n1;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        O[j][0] *= a0;
        O[j][1] *= a0;
        O[j][2] *= a1;
        O[j][3] *= a1;
      }
      lb[0] *= a0;
      lb[1] *= a0;
      lb[2] *= a1;
      lb[3] *= a1;
    }
    const float mu0 = m_ref[0] == -INFINITY ? 0.f : m_ref[0];
    const float mu1 = m_ref[1] == -INFINITY ? 0.f : m_ref[1];
    // ---- O += P V, one 16-token k-chunk (n-tiles 2 cc, 2 cc + 1) at a time
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t pa[4];
      float z[8];
      fma2(z[0], z[1], s[2 * cc][0], s[2 * cc][1], sl2, -mu0);
      fma2(z[2], z[3], s[2 * cc][2], s[2 * cc][3], sl2, -mu1);
      fma2(z[4], z[5], s[2 * cc + 1][0], s[2 * cc + 1][1], sl2, -mu0);
      fma2(z[6], z[7], s[2 * cc + 1][2], s[2 * cc + 1][3], sl2, -mu1);
#pragma unroll
      for (int k = 0; k < 4; ++k) pa[k] = pack_f16x2(fast_exp2(z[2 * k]), fast_exp2(z[2 * k + 1]));
      // token pairs (2t, 2t+1) and (2t+8, 2t+9) of the chunk; a pair row's 16-byte chunks are
      // stored XOR-swizzled by 2 (pair mod 4) = 2t, so a quarter-warp hits every bank once
      const int pa_ = 8 * cc + t4, pb_ = pa_ + 4;
      const int sw = (g8 ^ (t4 << 1)) << 4;
      const uint4 va = *reinterpret_cast<const uint4*>(st + kOffVc + pa_ * kD + sw);
      const uint4 vb = *reinterpret_cast<const uint4*>(st + kOffVc + pb_ * kD + sw);
      const uint8_t* vsc = st + kOffVs + g8 * kPage + 16 * cc + 2 * t4;
      uint32_t sa = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(vsc));
      uint32_t sb = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(vsc + 8));
      if (nvalid < kPage) {  // tokens past the history: zero scale, so their codes contribute nothing
        const int ta = 16 * cc + 2 * t4, tb = ta + 8;
        sa &= (ta < nvalid ? 0x0000ffffu : 0u) | (ta + 1 < nvalid ? 0xffff0000u : 0u);
        sb &= (tb < nvalid ? 0x0000ffffu : 0u) | (tb + 1 < nvalid ? 0xffff0000u : 0u);
      }
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
      const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int wq = 0; wq < 4; ++wq) {
        uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
        e2m1x4_to_f16x2(wa[wq], a0, a1, a2, a3);
        e2m1x4_to_f16x2(wb[wq], c0, c1, c2, c3);
        mma_f16_16816(O[4 * wq + 0], pa, hmul2(a0, sa), hmul2(c0, sb));
        mma_f16_16816(O[4 * wq + 1], pa, hmul2(a1, sa), hmul2(c1, sb));
        mma_f16_16816(O[4 * wq + 2], pa, hmul2(a2, sa), hmul2(c2, sb));
        mma_f16_16816(O[4 * wq + 3], pa, hmul2(a3, sa), hmul2(c3, sb));
      }
      mma_f16_16816(lb, pa, kOnes, kOnes);
    }
  };

  reset_state();
  int u = u_first;
  int j = 0;       // own pages gone through
  int waited = 0;  // own pages whose loads are known to have landed
  while (true) {
    const long long seg_lo = max(g_begin, (long long)pre[u]);
    const long long seg_hi = min(g_end, (long long)pre[u + 1]);
    enter_unit(u);
    // this warp's pages of the segment: g = g_begin + warp (mod kWarps)
    const long long off = (seg_lo - g_begin) % kWarps;
    for (long long g = seg_lo + ((warp - off + kWarps) % kWarps); g < seg_hi; g += kWarps, ++j) {
      if ((j & 31) == 0 && j > 0) {  // next batch of page ids (resolved one batch ahead)
        ids_cur = ids_nxt;
        ids_nxt = resolve((j >> 5) + 1);
      }
      const int id = __shfl_sync(0xffffffffu, ids_cur, j & 31);
      const int slot = 2 * warp + (j & 1);
      if (!dead) {
        if (__all_sync(0xffffffffu, mbar_wait(&tail->full[slot], (j >> 1) & 1))) {
          waited = j + 1;
        } else {
          if (lane == 0) raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
          dead = true;  // stop loading; the loads in flight are waited for before the exit
        }
      }
      if (!dead) {
        const int nvalid = min(kPage, len_u - (int)(g - pre[u]) * kPage);
        if (id >= 0 && nvalid > 0) process_page(stages + (size_t)slot * kStageBytes, nvalid);
        __syncwarp();
        if (issued < n_own) {  // refill the slot with own page j + 2
          const int jn = issued;
          int src = ids_cur;
          if ((jn >> 5) != (j >> 5)) src = ids_nxt;  // only then wait for the next batch's ids
          issue(jn, __shfl_sync(0xffffffffu, src, jn & 31));
          ++issued;
        }
      }
    }

    // ---- end of a segment: merge the 8 warps, then write the unit or a segment record ----
    float lb0 = lb[0], lb1 = lb[2];  // the ones-column MMA leaves the row sum in every column
    if (t4 == 0) {
      tail->mstat[warp][g8] = m_ref[0];
      tail->mstat[warp][g8 + 8] = m_ref[1];
      tail->lstat[warp][g8] = lb0;
      tail->lstat[warp][g8 + 8] = lb1;
    }
    named_barrier_sync(1, kWarps * 32);
    {
      float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        M0 = fmaxf(M0, tail->mstat[w][g8]);
        M1 = fmaxf(M1, tail->mstat[w][g8 + 8]);
      }
      const float a0 = fast_exp2(m_ref[0] - (M0 == -INFINITY ? 0.f : M0));
      const float a1 = fast_exp2(m_ref[1] - (M1 == -INFINITY ? 0.f : M1));
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        O[j][0] *= a0;
        O[j][1] *= a0;
        O[j][2] *= a1;
        O[j][3] *= a1;
      }
    }
    {
      // fixed-order sum of the 8 warps' O (bit-reproducible): 4,5 -> 0,1; 6,7 -> 2,3; 2,3 -> 0,1;
      // 1 -> 0, through two fragment-layout slots
      auto put = [&](int slot) {
        float* dst = Obuf + slot * kRows * kD;
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[(j * 4 + e) * 32 + lane] = O[j][e];
      };
      auto add = [&](int slot) {
        const float* src = Obuf + slot * kRows * kD;
#pragma unroll
        for (int j = 0; j < 16; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) O[j][e] += src[(j * 4 + e) * 32 + lane];
      };
      const int cw = warp;
      if (cw == 4 || cw == 5) put(cw - 4);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 0 || cw == 1) add(cw);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 6 || cw == 7) put(cw - 6);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 2 || cw == 3) add(cw - 2);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 2 || cw == 3) put(cw - 2);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 0 || cw == 1) add(cw);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 1) put(1);
      named_barrier_sync(1, kWarps * 32);
      if (cw == 0) {
        add(1);
#pragma unroll
        for (int j = 0; j < 16; ++j) {  // natural [row][column] layout into slot 0
          const int ca = 32 * t4 + j, cb = ca + 16;
          float* r0 = Obuf + g8 * kD;
          r0[ca] = O[j][0];
          r0[cb] = O[j][1];
          r0[8 * kD + ca] = O[j][2];
          r0[8 * kD + cb] = O[j][3];
        }
      }
    }
    named_barrier_sync(1, kWarps * 32);

    // every consumer thread owns row r, columns [c0, c0 + 8)
    const int r = tid / 16;
    const int c0 = (tid % 16) * (kD / 16);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, tail->mstat[w][r]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float LB = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) LB += tail->lstat[w][r] * fast_exp2(tail->mstat[w][r] - Mu);

    const size_t orow = ((size_t)s_u * p.B + b_u) * p.Hq + (size_t)k_u * p.G + r;
    const bool whole = seg_lo == pre[u] && seg_hi == pre[u + 1];
    bool unit_written = whole;  // this CTA wrote the unit's final O_partial / lse
    if (whole) {
      if (r < p.G) {
        const float inv = LB > 0.f ? 1.f / LB : 0.f;
        float* dst = p.o_part + orow * kD + c0;
#pragma unroll
        for (int c = 0; c < kD / 16; c += 4)
          *reinterpret_cast<float4*>(dst + c) =
              make_float4(Obuf[r * kD + c0 + c] * inv, Obuf[r * kD + c0 + c + 1] * inv,
                          Obuf[r * kD + c0 + c + 2] * inv, Obuf[r * kD + c0 + c + 3] * inv);
        if (c0 == 0) p.lse[orow] = LB > 0.f ? (M + log2f(LB)) * kLn2 : -INFINITY;
      }
    } else {
      const int slot = (g_begin >= pre[u]) ? 0 : 1;
      float* rec = p.seg + ((size_t)blockIdx.x * 2 + slot) * kRec;
#pragma unroll
      for (int c = 0; c < kD / 16; c += 4)
        *reinterpret_cast<float4*>(rec + r * kD + c0 + c) =
            make_float4(Obuf[r * kD + c0 + c], Obuf[r * kD + c0 + c + 1],
                        Obuf[r * kD + c0 + c + 2], Obuf[r * kD + c0 + c + 3]);
      if (c0 == 0) {
        rec[kRows * kD + r] = M;
        rec[kRows * kD + 2 * kRows + r] = LB;
      }
      __threadfence();
      named_barrier_sync(1, kWarps * 32);
      const int c_lo = cta_of(pre[u], W, Geff);
      const int c_hi = cta_of((long long)pre[u + 1] - 1, W, Geff);
      if (tid == 0) {
        const int ticket = atomicAdd(&p.tickets[u], 1);
        tail->flag = (ticket == c_hi - c_lo) ? 1 : 0;
      }
      named_barrier_sync(1, kWarps * 32);
      unit_written = tail->flag != 0;
      if (tail->flag) {  // last arriver merges every segment of this unit
        __threadfence();
        float Mm = -INFINITY;
        for (int c = c_lo; c <= c_hi; ++c) {
          const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
          Mm = fmaxf(Mm, __ldcg(p.seg + ((size_t)c * 2 + sl) * kRec + kRows * kD + r));
        }
        const float Mmu = Mm == -INFINITY ? 0.f : Mm;
        float acc[kD / 16];
#pragma unroll
        for (int c = 0; c < kD / 16; ++c) acc[c] = 0.f;
        float LBm = 0.f;
        for (int c = c_lo; c <= c_hi; ++c) {
          const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
          const float* rc = p.seg + ((size_t)c * 2 + sl) * kRec;
          const float wgt = fast_exp2(__ldcg(rc + kRows * kD + r) - Mmu);
          LBm += __ldcg(rc + kRows * kD + 2 * kRows + r) * wgt;
#pragma unroll
          for (int cc = 0; cc < kD / 16; cc += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(rc + r * kD + c0 + cc));
            acc[cc] += v.x * wgt;
            acc[cc + 1] += v.y * wgt;
            acc[cc + 2] += v.z * wgt;
            acc[cc + 3] += v.w * wgt;
          }
        }
        if (r < p.G) {
          const float inv = LBm > 0.f ? 1.f / LBm : 0.f;
          float* dst = p.o_part + orow * kD + c0;
#pragma unroll
          for (int c = 0; c < kD / 16; c += 4)
            *reinterpret_cast<float4*>(dst + c) =
                make_float4(acc[c] * inv, acc[c + 1] * inv, acc[c + 2] * inv, acc[c + 3] * inv);
          if (c0 == 0) p.lse[orow] = LBm > 0.f ? (Mm + log2f(LBm)) * kLn2 : -INFINITY;
        }
        if (tid == 0) p.tickets[u] = 0;  // ready for the next launch
      }
    }
    if (p.o_out != nullptr && unit_written)
      fused_group_combine(p, (int)((u + p.u0) / p.kvp), &tail->gflag,
                          [] { named_barrier_sync(1, kWarps * 32); }, tid, warp, lane, kWarps);
    named_barrier_sync(1, kWarps * 32);
    reset_state();
    if (seg_hi >= g_end) break;
    do { ++u; } while (pre[u + 1] <= seg_hi);  // next unit with pages (skips empty units)
  }
  if (dead && lane == 0) {  // a wait gave up: let this warp's loads still in flight land first
    for (int jj = waited; jj < issued; ++jj)
      mbar_wait(&tail->full[2 * warp + (jj & 1)], (jj >> 1) & 1);
  }
}

}  // namespace

size_t gqa_nvfp4_smem_bytes(int units) { return smem_fixed() + (size_t)(units + 1) * sizeof(int); }

size_t gqa_nvfp4_segment_record_floats() { return kRec; }

helix_status gqa_partial_nvfp4_launch(const GqaParams& p, int grid, cudaStream_t stream) {
  if (p.D != kD) return HELIX_ERR_UNSUPPORTED;
  const size_t smem = gqa_nvfp4_smem_bytes(p.units);
  if (allow_max_dynamic_smem(reinterpret_cast<const void*>(gqa_partial_nvfp4_kernel)) !=
      cudaSuccess)
    return HELIX_ERR_CUDA;
  gqa_partial_nvfp4_kernel<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? HELIX_OK : HELIX_ERR_CUDA;
}

}  // namespace helix
