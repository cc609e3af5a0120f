// gqa_partial.cu -- per-shard partial decode attention for grouped-query attention over a bf16 KV
// cache (the NVFP4 cache has its own kernel, gqa_partial_nvfp4.cu).
//
// What it computes (paper summary "Helix Parallelism: Rethinking Sharding Strategies for
// Interactive Multi-Million-Token LLM Decoding", fdeinterviews.com, paragraph on KV parallelism):
// for every request b, KV head k and KVP shard s, over the tokens T_s the shard holds,
//     z_{h,t} = scale * <q_{b,h}, K_{t,k}>            for the G query heads h of KV head k
//     O_s[h]  = sum_t e^{z_{h,t} - m} V_{t,k} / sum_t e^{z_{h,t} - m},   lse_s[h] = m + ln sum_t ...
// The G heads of a group are the M = 16 rows of one m16n8k16 tensor-core tile, so the shard's K and V
// rows stream from HBM exactly once for all heads that share them.
//
// Work decomposition ("stream-K" over pages): the (b, k, s) units are laid end to end as one list
// of 64-token pages; each persistent CTA takes an equal contiguous range of that list, whatever the
// per-request lengths are. A CTA that finishes a unit inside its range writes the normalised result
// directly; a unit cut by range boundaries is written as unnormalised segments to the workspace and
// merged by whichever CTA arrives last on the unit's ticket (an atomic counter -- nobody spins).
//
// CTA layout: warps 0-7 are two consumer warpgroups that take alternate pages; warp w of a group owns
// tokens [16w, 16w+16) of its page. Warp 8 is the producer: it resolves the page ids of 32 pages at a
// time with one coalesced load, and one lane issues the loads of each page into an NSTAGE-deep ring
// guarded by mbarriers. NSTAGE is a multiple of the number of groups, so a stage is only ever used by
// one group and no consumer can wait on a phase more than one ahead of the one it last consumed.
// Softmax is online in fp32 and base 2 (scale * log2 e folded into the logits).
//
// K and V stream in with TMA tile loads of the page's rows (128-byte swizzle, 8 KiB per 64-column
// half); ldmatrix feeds the S = q K^T and P V tiles.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "combine_row.cuh"
#include "device_common.cuh"
#include "internal.h"

namespace helix {
namespace {

constexpr int kPage = 64;          // tokens per page
constexpr int kRows = 16;          // query-head rows per tile (G <= 16, zero-padded)
constexpr int kConsumerWarps = 8;  // two warpgroups
constexpr int kGroups = 2;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kChunkBytes = kPage * 64 * 2;  // one 64-column half of a bf16 page-head: 8 KiB
constexpr int kMergeSlots = 2;               // 16 x D fp32 buffers for the cross-warp merge
constexpr int kMinPagesPerCta = 4;

template <int D>
struct GqaCfg {
  static constexpr int NCH = D / 64;  // 64-column halves per bf16 row
  static constexpr int STAGE_BYTES = 2 * NCH * kChunkBytes;  // K and V of one (page, kv head)
  static constexpr int NSTAGE = D == 128 ? 6 : 10;
  // floats per workspace segment record: O [16][D], then m, l, lb per row
  static constexpr int REC = kRows * (D + 3);
  static_assert(NSTAGE % kGroups == 0, "a stage must belong to one consumer group");
  static_assert(NSTAGE <= 16, "SmemTail holds 16 barrier pairs");
};

struct SmemTail {
  uint64_t full[16];
  uint64_t empty[16];
  int stage_ok[16];  // written by the producer before it completes a stage: 1 = page loaded
  float mstat[kConsumerWarps][kRows];
  float lstat[kConsumerWarps][kRows];
  float lbstat[kConsumerWarps][kRows];
  int flag;
  int gflag;
  int abort_;
};

template <int D>
__host__ __device__ constexpr size_t smem_bytes_for(int units) {
  return 1024 /*alignment slack*/ + (size_t)GqaCfg<D>::NSTAGE * GqaCfg<D>::STAGE_BYTES +
         (size_t)kMergeSlots * kRows * D * sizeof(float) + sizeof(SmemTail) +
         (size_t)(units + 1) * sizeof(int);
}

__device__ __forceinline__ long long range_begin(int c, long long W, int G) {
  return (long long)c * W / G;
}
// CTA whose range holds page x (0 <= x < W), for ranges begin(c) = floor(c W / G) with G <= W.
__device__ __forceinline__ int cta_of(long long x, long long W, int G) {
  return (int)(((x + 1) * (long long)G - 1) / W);
}

// Warp-collective pipeline wait: every lane observes the phase itself (so each lane's later shared
// memory reads are ordered after the asynchronous writes the phase covers); false on timeout.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    gqa_partial_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const GqaParams p) {
  using Cfg = GqaCfg<D>;
  constexpr int NCH = Cfg::NCH;
  constexpr int NSTAGE = Cfg::NSTAGE;
  constexpr int KSTEPS = D / 16;  // k-steps of the QK^T contraction
  constexpr int NT = D / 8;       // n-tiles of the PV output

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* Obuf = reinterpret_cast<float*>(smem + (size_t)NSTAGE * Cfg::STAGE_BYTES);
  SmemTail* tail = reinterpret_cast<SmemTail*>(Obuf + kMergeSlots * kRows * D);
  int* pre = reinterpret_cast<int*>(tail + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int U = p.units;

  // ---- per-unit page counts and their prefix sums (every CTA computes the same table) ----
  for (int u = tid; u < U; u += kThreads) {
    const int s = (u + p.u0) % p.kvp;
    const int b = ((u + p.u0) / p.kvp) / p.Hkv;
    int len = p.shard_lens[s * p.B + b];
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
    tail->abort_ = 0;
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&tail->full[i], 1);
      mbar_init(&tail->empty[i], 4);
      tail->stage_ok[i] = 0;
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of pre[1..U], 32 lanes x contiguous chunks
    const int per = (U + 31) / 32;
    const int lo = 1 + lane * per, hi = min(U + 1, lo + per);
    int run = 0;
    for (int i = lo; i < hi; ++i) run += pre[i];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
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
  // Units with no tokens: O_s = 0, lse_s = -inf (handled round-robin by CTA index).
  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    if (pre[u + 1] != pre[u]) continue;
    const int s = (u + p.u0) % p.kvp, bk = (u + p.u0) / p.kvp, k = bk % p.Hkv, b = bk / p.Hkv;
    const size_t row0 = ((size_t)s * p.B + b) * p.Hq + (size_t)k * p.G;
    for (int i = tid; i < p.G * D; i += kThreads) p.o_part[row0 * D + i] = 0.f;
    for (int i = tid; i < p.G; i += kThreads) p.lse[row0 + i] = -INFINITY;
    if (p.o_out != nullptr)
      fused_group_combine(p, bk, &tail->gflag, [] { __syncthreads(); }, tid, warp, lane,
                          kThreads / 32);
  }
  // at least kMinPagesPerCta pages per CTA: short histories would otherwise be cut into one-page
  // pieces whose merges cost more than the pages (measured on the 4K-token workload)
  const int Geff = (int)min((long long)gridDim.x, (W + kMinPagesPerCta - 1) / kMinPagesPerCta);
  if ((int)blockIdx.x >= Geff) return;
  const long long g_begin = range_begin(blockIdx.x, W, Geff);
  const long long g_end = range_begin(blockIdx.x + 1, W, Geff);
  // first unit: pre[u] <= g_begin < pre[u+1]
  int u_first;
  {
    int lo = 0, hi = U;  // find the last u with pre[u] <= g_begin
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (pre[mid] <= g_begin) lo = mid; else hi = mid;
    }
    u_first = lo;
    while (pre[u_first + 1] <= g_begin) ++u_first;
  }

  // ======================================= producer =============================================
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
    }
    int u_cur = u_first;  // unit of the first page of the current batch (same in every lane)
    int stage = 0;
    uint32_t round = 0;
    long long issued = 0;
    bool dead = false;
    for (long long gb = g_begin; gb < g_end && !dead; gb += 32) {
      // each lane resolves page gb + lane: its unit, KV head and pool page id (one coalesced load)
      const long long gl = gb + lane;
      int my_page = -1, my_k = 0, uu = u_cur;
      if (gl < g_end) {
        while (pre[uu + 1] <= gl) ++uu;
        const int s = (uu + p.u0) % p.kvp, bk = (uu + p.u0) / p.kvp, b = bk / p.Hkv;
        my_k = bk % p.Hkv;
        my_page = __ldg(p.page_table + ((size_t)s * p.B + b) * p.max_pages + (int)(gl - pre[uu]));
      }
      const int nb = (int)min(32LL, g_end - gb);
      u_cur = __shfl_sync(0xffffffffu, uu, nb - 1);
      for (int j = 0; j < nb; ++j) {
        const int page = __shfl_sync(0xffffffffu, my_page, j);
        const int k = __shfl_sync(0xffffffffu, my_k, j);
        if (lane == 0 && !dead) {
          if (*(volatile int*)&tail->abort_) {
            dead = true;
          } else if (round > 0 && !mbar_wait(&tail->empty[stage], (round - 1) & 1)) {
            raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
            *(volatile int*)&tail->abort_ = 1;
            dead = true;
          } else {
            uint8_t* st = stages + (size_t)stage * Cfg::STAGE_BYTES;
            if (page < 0 || page >= p.num_pages) {
              raise_dev_error(p.err, HELIX_DEVERR_PAGE_ID);
              tail->stage_ok[stage] = 0;
              mbar_arrive(&tail->full[stage]);  // completes the phase with no data
            } else {
              tail->stage_ok[stage] = 1;
              mbar_arrive_expect_tx(&tail->full[stage], Cfg::STAGE_BYTES);
              const int row = (page * p.Hkv + k) * kPage;
#pragma unroll
              for (int c = 0; c < NCH; ++c) {
                tma_load_2d(st + c * kChunkBytes, &tmK, c * 64, row, &tail->full[stage]);
                tma_load_2d(st + (NCH + c) * kChunkBytes, &tmV, c * 64, row, &tail->full[stage]);
              }
            }
            ++issued;
            if (++stage == NSTAGE) { stage = 0; ++round; }
          }
        }
        dead = __shfl_sync(0xffffffffu, dead ? 1 : 0, 0) != 0;
      }
    }
    if (dead && lane == 0) {  // let every load already issued land before the CTA exits
      for (long long j = issued > NSTAGE ? issued - NSTAGE : 0; j < issued; ++j)
        mbar_wait(&tail->full[j % NSTAGE], (uint32_t)((j / NSTAGE) & 1));
    }
    return;
  }

  // ======================================= consumers ============================================
  const int grp = warp / 4;   // which warpgroup: takes pages i with i % 2 == grp
  const int w4 = warp & 3;    // token slice [16 w4, 16 w4 + 16) of the page
  const int g8 = lane >> 2;   // fragment row (query head) g and g + 8
  const int t4 = lane & 3;
  const int tok0 = 16 * w4;
  const int mi = lane >> 3, r8 = lane & 7;  // ldmatrix: which 8x8 matrix this lane addresses

  uint32_t qa[KSTEPS][4];
  float O[NT][4];
  // m: running max (base-2 logits); l: sum of fp32 weights (for the LSE); lb: sum of the rounded
  // weights the tensor cores multiply V by (normalises O, so O stays a convex combination of V rows)
  float m_run[2], l_run[2], lb_run[2];
  auto reset_state = [&]() {
#pragma unroll
    for (int j = 0; j < NT; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
    lb_run[0] = lb_run[1] = 0.f;
  };
  auto load_q = [&](int u) {
    const int bk = (u + p.u0) / p.kvp, k = bk % p.Hkv, b = bk / p.Hkv;
    const __nv_bfloat16* qb = p.q + ((size_t)b * p.Hq + (size_t)k * p.G) * D;
    const bool v0 = g8 < p.G, v1 = g8 + 8 < p.G;
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qb + (size_t)g8 * D);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(qb + (size_t)(g8 + 8) * D);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int c0 = 16 * kk + 2 * t4;
      qa[kk][0] = v0 ? __ldg(r0 + c0 / 2) : 0u;
      qa[kk][1] = v1 ? __ldg(r1 + c0 / 2) : 0u;
      qa[kk][2] = v0 ? __ldg(r0 + (c0 + 8) / 2) : 0u;
      qa[kk][3] = v1 ? __ldg(r1 + (c0 + 8) / 2) : 0u;
    }
  };

  reset_state();
  int u = u_first;
  int s_u = 0, b_u = 0, k_u = 0, len_u = 0;
  auto enter_unit = [&](int uu) {
    s_u = (uu + p.u0) % p.kvp;
    const int bk = (uu + p.u0) / p.kvp;
    k_u = bk % p.Hkv;
    b_u = bk / p.Hkv;
    len_u = p.shard_lens[s_u * p.B + b_u];
    load_q(uu);
  };
  enter_unit(u);
  long long seg_begin = g_begin;
  bool dead = false;
  int stage = 0, parity = 0, gsel = 0;
  const float sl2 = p.scale_log2;

  for (long long g = g_begin; g < g_end; ++g) {
    if (pre[u + 1] <= g) {  // entered a new unit
      while (pre[u + 1] <= g) ++u;
      enter_unit(u);
    }
    const int pg = (int)(g - pre[u]);
    if (gsel == grp) {
      if (!dead && *(volatile int*)&tail->abort_) dead = true;
      if (!dead && !warp_wait(&tail->full[stage], parity)) {
        if (lane == 0) {
          raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
          *(volatile int*)&tail->abort_ = 1;
        }
        dead = true;
      }
      if (!dead) {
        const int nvalid = min(kPage, len_u - pg * kPage);
        uint8_t* st = stages + (size_t)stage * Cfg::STAGE_BYTES;
        if (tail->stage_ok[stage] && tok0 < nvalid) {
          float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
          const uint32_t kbase = smem_u32(st);
          // zero the V rows past the end of the history in this warp's slice (0 * garbage = NaN)
          if (tok0 + 16 > nvalid) {
            for (int e = lane; e < 16 * NCH * 8; e += 32) {
              const int row = tok0 + e / (NCH * 8);
              const int rem = e % (NCH * 8);
              if (row >= nvalid)
                *reinterpret_cast<uint4*>(st + (NCH + rem / 8) * kChunkBytes + row * 128 +
                                          (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
          }
          {  // S = q K^T over this warp's 16 tokens: two n-tiles of 8 tokens
            const int token = tok0 + (mi >> 1) * 8 + r8;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
              const int dch = 2 * kk + (mi & 1);  // 16-byte column chunk of the row
              const uint32_t addr = kbase + (dch >> 3) * kChunkBytes + token * 128 +
                                    ((((dch & 7) ^ (token & 7))) << 4);
              uint32_t b0, b1, b2, b3;
              ldsm_x4(addr, b0, b1, b2, b3);
              mma_bf16_16816(s0, qa[kk], b0, b1);
              mma_bf16_16816(s1, qa[kk], b2, b3);
            }
          }
          // online softmax (base 2)
          const int ta = tok0 + 2 * t4, tb = tok0 + 8 + 2 * t4;
          float x[8];
          x[0] = ta < nvalid ? s0[0] * sl2 : -INFINITY;
          x[1] = ta + 1 < nvalid ? s0[1] * sl2 : -INFINITY;
          x[2] = tb < nvalid ? s1[0] * sl2 : -INFINITY;
          x[3] = tb + 1 < nvalid ? s1[1] * sl2 : -INFINITY;
          x[4] = ta < nvalid ? s0[2] * sl2 : -INFINITY;
          x[5] = ta + 1 < nvalid ? s0[3] * sl2 : -INFINITY;
          x[6] = tb < nvalid ? s1[2] * sl2 : -INFINITY;
          x[7] = tb + 1 < nvalid ? s1[3] * sl2 : -INFINITY;
          float mx0 = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
          float mx1 = fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7]));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
          const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
          const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
          const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
          const float al0 = fast_exp2(m_run[0] - mu0), al1 = fast_exp2(m_run[1] - mu1);
          m_run[0] = mn0;
          m_run[1] = mn1;
          float pw[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) pw[e] = fast_exp2(x[e] - mu0);
#pragma unroll
          for (int e = 4; e < 8; ++e) pw[e] = fast_exp2(x[e] - mu1);
          l_run[0] = l_run[0] * al0 + ((pw[0] + pw[1]) + (pw[2] + pw[3]));
          l_run[1] = l_run[1] * al1 + ((pw[4] + pw[5]) + (pw[6] + pw[7]));
          uint32_t pa[4];
          pa[0] = pack_bf16x2(pw[0], pw[1]);  // row g,   k 2t..
          pa[1] = pack_bf16x2(pw[4], pw[5]);  // row g+8, k 2t..
          pa[2] = pack_bf16x2(pw[2], pw[3]);  // row g,   k 8+2t..
          pa[3] = pack_bf16x2(pw[6], pw[7]);  // row g+8, k 8+2t..
          lb_run[0] = lb_run[0] * al0 + (bf16_lo_to_f32(pa[0]) + bf16_hi_to_f32(pa[0])) +
                      (bf16_lo_to_f32(pa[2]) + bf16_hi_to_f32(pa[2]));
          lb_run[1] = lb_run[1] * al1 + (bf16_lo_to_f32(pa[1]) + bf16_hi_to_f32(pa[1])) +
                      (bf16_lo_to_f32(pa[3]) + bf16_hi_to_f32(pa[3]));
          if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              O[j][0] *= al0;
              O[j][1] *= al0;
              O[j][2] *= al1;
              O[j][3] *= al1;
            }
          }
          // O += P V over the 16 tokens: V^T fragments via transposing ldmatrix
          const uint32_t vbase = smem_u32(st) + NCH * kChunkBytes;
          const int token = tok0 + (mi & 1) * 8 + r8;
#pragma unroll
          for (int n2 = 0; n2 < NT / 2; ++n2) {
            const int dch = 2 * n2 + (mi >> 1);
            const uint32_t addr = vbase + (dch >> 3) * kChunkBytes + token * 128 +
                                  ((((dch & 7) ^ (token & 7))) << 4);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_trans(addr, v0, v1, v2, v3);
            mma_bf16_16816(O[2 * n2], pa, v0, v1);
            mma_bf16_16816(O[2 * n2 + 1], pa, v2, v3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->empty[stage]);
      }
    }
    if (++gsel == kGroups) gsel = 0;
    if (++stage == NSTAGE) { stage = 0; parity ^= 1; }

    // ---- end of a segment: the unit ends here or the CTA's range does ----
    if (g + 1 == g_end || g + 1 == pre[u + 1]) {
      const int cw = warp;  // consumer warp 0..7
      float l0 = l_run[0], l1 = l_run[1];
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      float lb0 = lb_run[0], lb1 = lb_run[1];
      lb0 += __shfl_xor_sync(0xffffffffu, lb0, 1);
      lb0 += __shfl_xor_sync(0xffffffffu, lb0, 2);
      lb1 += __shfl_xor_sync(0xffffffffu, lb1, 1);
      lb1 += __shfl_xor_sync(0xffffffffu, lb1, 2);
      if (t4 == 0) {
        tail->mstat[cw][g8] = m_run[0];
        tail->mstat[cw][g8 + 8] = m_run[1];
        tail->lstat[cw][g8] = l0;
        tail->lstat[cw][g8 + 8] = l1;
        tail->lbstat[cw][g8] = lb0;
        tail->lbstat[cw][g8 + 8] = lb1;
      }
      named_barrier_sync(1, kConsumerWarps * 32);
      {
        float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          M0 = fmaxf(M0, tail->mstat[w][g8]);
          M1 = fmaxf(M1, tail->mstat[w][g8 + 8]);
        }
        const float a0 = fast_exp2(m_run[0] - (M0 == -INFINITY ? 0.f : M0));
        const float a1 = fast_exp2(m_run[1] - (M1 == -INFINITY ? 0.f : M1));
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          O[j][0] *= a0;
          O[j][1] *= a0;
          O[j][2] *= a1;
          O[j][3] *= a1;
        }
      }
      // Sum the 8 warps' O in a fixed order so results are bit-reproducible: warps 4..7 into
      // 0..3 (two at a time through the two merge slots), then 2,3 into 0,1, then 1 into 0.
      {
        auto put = [&](int slot) {
          float* dst = Obuf + slot * kRows * D;
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[(j * 4 + e) * 32 + lane] = O[j][e];
        };
        auto add = [&](int slot) {
          const float* src = Obuf + slot * kRows * D;
#pragma unroll
          for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) O[j][e] += src[(j * 4 + e) * 32 + lane];
        };
        // (writer warps, reader warps): (4,5 -> 0,1), (6,7 -> 2,3), (2,3 -> 0,1), (1 -> 0)
        if (cw == 4 || cw == 5) put(cw - 4);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 0 || cw == 1) add(cw);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 6 || cw == 7) put(cw - 6);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 2 || cw == 3) add(cw - 2);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 2 || cw == 3) put(cw - 2);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 0 || cw == 1) add(cw);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 1) put(1);
        named_barrier_sync(1, kConsumerWarps * 32);
        if (cw == 0) {
          add(1);
#pragma unroll
          for (int j = 0; j < NT; ++j) {  // natural [row][column] layout into slot 0
            // n-tile j, fragment columns 2t, 2t+1 are head-dim columns 8j + 2t (+1)
            const int ca = 8 * j + 2 * t4;
            const int cb = ca + 1;
            float* r0 = Obuf + g8 * D;
            r0[ca] = O[j][0];
            r0[cb] = O[j][1];
            r0[8 * D + ca] = O[j][2];
            r0[8 * D + cb] = O[j][3];
          }
        }
      }
      named_barrier_sync(1, kConsumerWarps * 32);

      // every consumer thread owns row r, columns [c0, c0 + D/16)
      const int r = tid / 16;
      const int c0 = (tid % 16) * (D / 16);
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, tail->mstat[w][r]);
      const float Mu = M == -INFINITY ? 0.f : M;
      float L = 0.f, LB = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float e = fast_exp2(tail->mstat[w][r] - Mu);
        L += tail->lstat[w][r] * e;
        LB += tail->lbstat[w][r] * e;
      }

      const size_t orow = ((size_t)s_u * p.B + b_u) * p.Hq + (size_t)k_u * p.G + r;
      const bool whole = seg_begin == pre[u] && g + 1 == pre[u + 1];
      bool unit_written = whole;  // this CTA wrote the unit's final O_partial / lse
      if (whole) {
        if (r < p.G) {
          const float inv = LB > 0.f ? 1.f / LB : 0.f;
          float* dst = p.o_part + orow * D + c0;
#pragma unroll
          for (int c = 0; c < D / 16; c += 4)
            *reinterpret_cast<float4*>(dst + c) =
                make_float4(Obuf[r * D + c0 + c] * inv, Obuf[r * D + c0 + c + 1] * inv,
                            Obuf[r * D + c0 + c + 2] * inv, Obuf[r * D + c0 + c + 3] * inv);
          if (c0 == 0) p.lse[orow] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
        }
      } else {
        const int slot = (g_begin >= pre[u]) ? 0 : 1;
        float* rec = p.seg + ((size_t)blockIdx.x * 2 + slot) * Cfg::REC;
#pragma unroll
        for (int c = 0; c < D / 16; c += 4) {
          *reinterpret_cast<float4*>(rec + r * D + c0 + c) =
              make_float4(Obuf[r * D + c0 + c], Obuf[r * D + c0 + c + 1],
                          Obuf[r * D + c0 + c + 2], Obuf[r * D + c0 + c + 3]);
        }
        if (c0 == 0) {
          rec[kRows * D + r] = M;
          rec[kRows * D + kRows + r] = L;
          rec[kRows * D + 2 * kRows + r] = LB;
        }
        __threadfence();
        named_barrier_sync(1, kConsumerWarps * 32);
        const int c_lo = cta_of(pre[u], W, Geff);
        const int c_hi = cta_of((long long)pre[u + 1] - 1, W, Geff);
        if (tid == 0) {
          const int ticket = atomicAdd(&p.tickets[u], 1);
          tail->flag = (ticket == c_hi - c_lo) ? 1 : 0;
        }
        named_barrier_sync(1, kConsumerWarps * 32);
        unit_written = tail->flag != 0;
        if (tail->flag) {  // last arriver merges every segment of this unit
          __threadfence();
          float Mm = -INFINITY;
          for (int c = c_lo; c <= c_hi; ++c) {
            const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
            const float* rc = p.seg + ((size_t)c * 2 + sl) * Cfg::REC;
            Mm = fmaxf(Mm, __ldcg(rc + kRows * D + r));
          }
          const float Mmu = Mm == -INFINITY ? 0.f : Mm;
          float acc[D / 16];
#pragma unroll
          for (int c = 0; c < D / 16; ++c) acc[c] = 0.f;
          float Lm = 0.f, LBm = 0.f;
          for (int c = c_lo; c <= c_hi; ++c) {
            const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
            const float* rc = p.seg + ((size_t)c * 2 + sl) * Cfg::REC;
            const float wgt = fast_exp2(__ldcg(rc + kRows * D + r) - Mmu);
            Lm += __ldcg(rc + kRows * D + kRows + r) * wgt;
            LBm += __ldcg(rc + kRows * D + 2 * kRows + r) * wgt;
#pragma unroll
            for (int cc = 0; cc < D / 16; cc += 4) {
              const float4 v = __ldcg(reinterpret_cast<const float4*>(rc + r * D + c0 + cc));
              acc[cc] += v.x * wgt;
              acc[cc + 1] += v.y * wgt;
              acc[cc + 2] += v.z * wgt;
              acc[cc + 3] += v.w * wgt;
            }
          }
          if (r < p.G) {
            const float inv = LBm > 0.f ? 1.f / LBm : 0.f;
            float* dst = p.o_part + orow * D + c0;
#pragma unroll
            for (int c = 0; c < D / 16; c += 4)
              *reinterpret_cast<float4*>(dst + c) =
                  make_float4(acc[c] * inv, acc[c + 1] * inv, acc[c + 2] * inv, acc[c + 3] * inv);
            if (c0 == 0) p.lse[orow] = Lm > 0.f ? (Mm + log2f(Lm)) * kLn2 : -INFINITY;
          }
          if (tid == 0) p.tickets[u] = 0;  // ready for the next launch
        }
      }
      if (p.o_out != nullptr && unit_written)
        fused_group_combine(p, (int)((u + p.u0) / p.kvp), &tail->gflag,
                            [] { named_barrier_sync(1, kConsumerWarps * 32); }, tid, warp, lane,
                            kConsumerWarps);
      named_barrier_sync(1, kConsumerWarps * 32);
      reset_state();
      seg_begin = g + 1;
    }
  }
}

}  // namespace

template <int D>
static helix_status launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const GqaParams& p,
                           int grid, cudaStream_t stream) {
  const size_t smem = smem_bytes_for<D>(p.units);
  auto kern = gqa_partial_kernel<D>;
  if (allow_max_dynamic_smem(reinterpret_cast<const void*>(kern)) != cudaSuccess)
    return HELIX_ERR_CUDA;
  kern<<<grid, kThreads, smem, stream>>>(tmK, tmV, p);
  return cudaGetLastError() == cudaSuccess ? HELIX_OK : HELIX_ERR_CUDA;
}

size_t gqa_partial_smem_bytes(int head_dim, int units) {
  return head_dim == 64 ? smem_bytes_for<64>(units) : smem_bytes_for<128>(units);
}

size_t gqa_segment_record_floats(int head_dim) {
  return head_dim == 64 ? GqaCfg<64>::REC : GqaCfg<128>::REC;
}

helix_status gqa_partial_bf16_launch(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                     const GqaParams& p, int grid, cudaStream_t stream) {
  if (p.D == 128) return launch<128>(tmK, tmV, p, grid, stream);
  if (p.D == 64) return launch<64>(tmK, tmV, p, grid, stream);
  return HELIX_ERR_UNSUPPORTED;
}

}  // namespace helix
