// mla_partial.cu -- per-shard partial decode attention for absorbed multi-head latent attention
// (MLA) on the 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes: 128 query heads attend to ONE shared latent KV head (the paper summary's
// tensor-parallelism paragraph notes that MLA "effectively" has one KV head, which is why its KV
// cannot be split by heads and KV parallelism is needed). With the absorbed formulation the latent
// row c_t (576 wide) is the key and its first 512 columns are the value:
//     z_{h,t} = scale * <q_h, c_t>,  O_s[h] = sum_t e^{z - m} c_t[0:512] / sum_t e^{z - m},
//     lse_s[h] = m + ln sum_t e^{z - m}
// over the tokens T_s of KVP shard s (paper summary, paragraph on KV parallelism).
//
// Sizes force a two-CTA design. O for 128 heads x 512 columns in fp32 fills all 512 TMEM columns
// and q (128 x 576 bf16) alone is 144 KiB, so one CTA cannot hold q, a score tile and O. A cluster
// of two CTAs works on the same 64-token tiles (one page each):
//   * CTA r takes half of the contraction, head-dim elements [288 r, 288 r + 288): four whole
//     64-column chunks of q in shared memory (chunks 0-3, or 5-8) and its 32 columns of the
//     shared chunk 4 in 16 TMEM columns (loaded by the softmax warps at each new request), and
//     computes a partial score tile S_r = q[:, half] C[:, half]^T (M = 128 heads, N = 64 tokens,
//     K = 288) into TMEM: 2 k-steps with A from TMEM, then 16 with both operands in shared memory.
//     A tcgen05.mma of M = 128 costs about the same for any N up to 128 (measured: about 110 SM
//     cycles for one K = 16 step), so the score tile is as wide as a page;
//   * the two CTAs swap their partials through distributed shared memory: st.async stores into the
//     peer's exchange buffer complete a transaction count on the peer's mbarrier, and the buffer is
//     handed back with a relaxed remote arrive (no multicast loads anywhere), so both hold the same
//     full S. One exchange buffer serves the tiles in turn;
//   * each CTA runs the same online softmax, writes P (bf16) back into TMEM and accumulates O for
//     its half of the value columns (M = 128, N = 256, K = 64 tokens) in 256 TMEM columns with the
//     TS form of the MMA (A = P from TMEM, B = V read straight from the latent tile it already holds,
//     MN-major).
// Each CTA loads five 64-column chunks of every latent row (chunks 0-4 or 4-8), so together the pair
// reads the 576-wide row once plus one 64-column chunk. With q's half chunk in TMEM, three 40 KiB
// tile stages fit beside q (64 KiB) and the exchange buffer: the load of a tile waits for the P V
// product three tiles back, which is what bounds the tile period (the chain of one tile: load,
// scores, exchange, softmax, P V, over the number of stages).
//
// Warps: 0-7 softmax / epilogue in two groups of four (group g takes the tiles i with i % 2 == g,
// so two tiles are in the softmax at once; thread h of a group owns head h = TMEM lane h), 8 TMA
// producer (and L2 prefetch one tile ahead), 9 score-MMA issuer and TMEM allocator, 10 P V issuer
// (one thread each, so a ready P V never waits behind a score tile). Each group has its own TMEM
// score buffer, so the tensor core computes the next tile's scores while a group works on its
// tile. The groups share one reference maximum per head, handed from the owner of tile i-1 to the
// owner of tile i through shared memory and an mbarrier per 32-row slice; each group keeps its own
// running sum, and the two are merged at the end of a segment. O is rescaled lazily: the exponent
// base only moves when a row maximum grows by more than 8 (in base-2 units), so weights stay below
// 2^8 and the 256-column TMEM rescale is rare. The logit scale is applied inside the exponent.
// Work is split over the (request, shard) units exactly as in the GQA kernel: each cluster takes an
// equal contiguous range of 64-token tiles; split units are merged by the last arriving cluster,
// per value half.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "device_common.cuh"
#include "internal.h"

namespace helix {
namespace {

constexpr int kHeads = 128;
constexpr int kDV = 512, kHalfDV = 256;  // V: the first 512 of the 576 latent columns
constexpr int kTok = 64;                   // tokens per tile (one page)
constexpr int kPageTok = 64;               // tokens per page
constexpr int kChunks = 5;                 // 64-column chunks of a latent row per CTA
constexpr int kQChunks = 4;                // full 64-column chunks of q per CTA (in shared memory)
constexpr int kKSteps = 18;                // 288 / 16: 2 over the half chunk, 16 over whole ones
static_assert(2 + 4 * kQChunks == kKSteps, "a CTA's 288 columns: four chunks and a half");
constexpr int kNS = 3;                     // tile stages
constexpr int kNX = 1;                     // score-exchange buffers (the groups take turns)
constexpr int kPrefetch = 1;               // tiles fetched into L2 ahead of the TMA loads
constexpr int kStageBytes = kTok * kChunks * 128;     // 40 KiB
constexpr int kQBytes = kHeads * kQChunks * 128;       // 64 KiB
constexpr int kSBuf = 2;                               // score-tile buffers in TMEM
constexpr uint32_t kSCol = 256, kPCol = 384;           // TMEM columns: O [0,256), S 2x64, P 2x32
// and q's 32 columns of the shared chunk (the half of columns 256..319 this CTA takes), 16 columns
// of bf16 pairs: the A operand of the two score k-steps over that half chunk
constexpr uint32_t kQhCol = 448;
// exchange buffer: [kTok / 4][kHeads] groups of four fp32 scores, so that the 32 rows of a warp
// write (remotely) and read 512 contiguous bytes per instruction
constexpr int kXBytes = kHeads * kTok * 4;             // 32 KiB
// warps 0-7: two softmax groups of four (group g takes the tiles i with i % 2 == g)
constexpr int kProducerWarp = 8, kMmaWarp = 9, kPvWarp = 10;
constexpr int kThreads = 11 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kRec = kHeads * (kHalfDV + 3);           // floats per segment record (one half)

struct MlaTail {
  uint64_t stage_full[kNS], stage_empty[kNS];
  uint64_t s_full[kSBuf], s_empty[kSBuf];
  uint64_t p_full[2], p_empty[2];
  uint64_t x_full[kNX], x_free[kNX];
  uint64_t q_full, q_empty;
  uint64_t qh_full;  // q's half chunk for the next unit is in TMEM (one arrival per warp of a group)
  int stage_ok[kNS];
  uint64_t m_ready[2][4];   // [publishing group][32-row slice]: mpub holds its latest maximum
  uint64_t seg_ready;       // segment end: the non-owning group has stored its (m, l)
  uint64_t o_drained;       // segment end: the owning group has read O out of TMEM
  float mpub[kHeads];       // reference maximum after the latest tile, handed between groups
  float seg_m[2][kHeads];   // per group: the maximum its running sum is relative to
  float seg_l[2][kHeads];   // per group: running sum of the weights of its tiles
  uint32_t tmem_base;
  int flag;
  int abort_;
};

constexpr size_t kSmemFixed = 1024 + kQBytes + kNS * kStageBytes + kNX * kXBytes +
                              sizeof(MlaTail);

// ------------------------------------------------------------------------------------------------
// tcgen05 / cluster helpers

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// shared::cluster address of the same variable in CTA `rank`
__device__ __forceinline__ uint32_t map_peer(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
// Relaxed remote arrival (no implicit cluster-scope fence). Used only to hand a buffer back after
// reading it; the caller makes the arrival depend on every loaded value first (keep_alive), so the
// loads have completed before the arrival can be issued.
__device__ __forceinline__ void remote_arrive_relaxed(uint32_t cluster_bar_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   cluster_bar_addr)
               : "memory");
}
template <int N>
__device__ __forceinline__ void keep_alive(const float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" ::"f"(v[i]));
}
// Asynchronous store into the peer CTA's shared memory; its completion counts `16` bytes against
// the transaction count of the peer's mbarrier (no fence needed on either side).
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d,
                                            uint32_t remote_bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::
          "r"(addr),
      "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
      : "memory");
}
// wait with cluster-scope acquire (data written by the peer CTA)
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
#pragma unroll 1
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D (+)= A B with A read from tensor memory (K-major: row m in lane m, two bf16 per column)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 64 consecutive fp32 columns of this thread's TMEM lane (two 32-column loads, one wait)
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
#pragma unroll
  for (int half = 0; half < 2; ++half)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[32 * half + 0]), "=r"(r[32 * half + 1]), "=r"(r[32 * half + 2]),
          "=r"(r[32 * half + 3]), "=r"(r[32 * half + 4]), "=r"(r[32 * half + 5]),
          "=r"(r[32 * half + 6]), "=r"(r[32 * half + 7]), "=r"(r[32 * half + 8]),
          "=r"(r[32 * half + 9]), "=r"(r[32 * half + 10]), "=r"(r[32 * half + 11]),
          "=r"(r[32 * half + 12]), "=r"(r[32 * half + 13]), "=r"(r[32 * half + 14]),
          "=r"(r[32 * half + 15]), "=r"(r[32 * half + 16]), "=r"(r[32 * half + 17]),
          "=r"(r[32 * half + 18]), "=r"(r[32 * half + 19]), "=r"(r[32 * half + 20]),
          "=r"(r[32 * half + 21]), "=r"(r[32 * half + 22]), "=r"(r[32 * half + 23]),
          "=r"(r[32 * half + 24]), "=r"(r[32 * half + 25]), "=r"(r[32 * half + 26]),
          "=r"(r[32 * half + 27]), "=r"(r[32 * half + 28]), "=r"(r[32 * half + 29]),
          "=r"(r[32 * half + 30]), "=r"(r[32 * half + 31])
        : "r"(taddr + 32 * half));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 consecutive 32-bit columns of this thread's TMEM lane (raw bits)
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
      "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
      "r"(v[30]), "r"(v[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 16 consecutive 32-bit columns of this thread's TMEM lane (raw bits)
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start, leading and stride byte offsets in
// 16-byte units, descriptor version 1, swizzle mode in the top three bits.
constexpr uint64_t kSwizzle128 = 2;
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint64_t swizzle) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (swizzle << 61);
}
// Instruction descriptor for kind::f16: fp32 accumulate, bf16 A and B, A K-major, B K-major or
// MN-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ long long range_begin(int c, long long W, int G) {
  return (long long)c * W / G;
}
__device__ __forceinline__ int cta_of(long long x, long long W, int G) {
  return (int)(((x + 1) * (long long)G - 1) / W);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_partial_kernel(const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmQ, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* q_s = smem;                                   // [4 chunks][128 rows][128 B]
  uint8_t* stage_s = q_s + kQBytes;                      // [kNS][5 chunks][64 rows][128 B]
  float* x_s = reinterpret_cast<float*>(stage_s + kNS * kStageBytes);  // [kNX][kTok/4][128][4]
  MlaTail* tail = reinterpret_cast<MlaTail*>(x_s + kNX * kHeads * kTok);
  int* pre = reinterpret_cast<int*>(tail + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int U = p.units;  // (b, s) units

  // ---- tiles per unit and their prefix sums ----
  for (int u = tid; u < U; u += kThreads) {
    const int s = (u + p.u0) % p.kvp, b = (u + p.u0) / p.kvp;
    int len = p.shard_lens[s * p.B + b];
    if (len > p.max_pages * kPageTok) {
      if (blockIdx.x == 0) raise_dev_error(p.err, HELIX_DEVERR_CAPACITY);
      len = p.max_pages * kPageTok;
    }
    pre[u + 1] = len > 0 ? (len + kTok - 1) / kTok : 0;
  }
  if (tid == 0) {
    pre[0] = 0;
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&tail->stage_full[i], 1);
      mbar_init(&tail->stage_empty[i], 1);
    }
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&tail->s_full[i], 1);
      mbar_init(&tail->s_empty[i], 4);  // one arrival per warp of the group that reads it
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tail->p_full[i], 4);
      mbar_init(&tail->p_empty[i], 1);
      for (int j = 0; j < 4; ++j) mbar_init(&tail->m_ready[i][j], 32);  // every lane of a warp
    }
    mbar_init(&tail->seg_ready, kHeads);  // every thread of a group
    mbar_init(&tail->o_drained, kHeads);
    for (int i = 0; i < kNX; ++i) {
      // x_full: armed by this CTA with the expected bytes, completed by the peer's async stores
      mbar_init(&tail->x_full[i], 1);
      mbar_init(&tail->x_free[i], 4);  // one arrival per warp of the peer CTA's group
    }
    mbar_init(&tail->q_full, 1);
    mbar_init(&tail->q_empty, 1);
    mbar_init(&tail->qh_full, 4);
    tail->flag = 0;
    tail->abort_ = 0;
    fence_mbar_init();
    // arm the exchange barrier for the first tile (128 rows x 64 fp32 scores)
    for (int i = 0; i < kNX; ++i) mbar_arrive_expect_tx(&tail->x_full[i], kHeads * kTok * 4);
  }
  if (warp == kMmaWarp) {  // allocate all 512 TMEM columns (one CTA per SM)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tail->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) {
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the peer's barriers are initialised before any remote arrival

  const uint32_t tmem = tail->tmem_base;
  const long long W = pre[U];
  // units with no tokens: O_s = 0, lse_s = -inf (this CTA's value half)
  for (int u = pair; u < U; u += npairs) {
    if (pre[u + 1] != pre[u]) continue;
    const int s = (u + p.u0) % p.kvp, b = (u + p.u0) / p.kvp;
    const size_t row0 = ((size_t)s * p.B + b) * kHeads;
    for (int i = tid; i < kHeads * kHalfDV; i += kThreads)
      p.o_part[(row0 + i / kHalfDV) * kDV + rank * kHalfDV + i % kHalfDV] = 0.f;
    if (rank == 0)
      for (int i = tid; i < kHeads; i += kThreads) p.lse[row0 + i] = -INFINITY;
  }
  const int Geff = (int)min((long long)npairs, W);
  const bool active = pair < Geff;
  const long long g_begin = active ? range_begin(pair, W, Geff) : 0;
  const long long g_end = active ? range_begin(pair + 1, W, Geff) : 0;
  int u_first = 0;
  if (active) {
    int lo = 0, hi = U;
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (pre[mid] <= g_begin) lo = mid; else hi = mid;
    }
    u_first = lo;
    while (pre[u_first + 1] <= g_begin) ++u_first;
  }

  if (warp == kProducerWarp) {
    // ===================================== TMA producer ========================================
    if (lane == 0 && active) {
      prefetch_tensormap(&tmC);
      prefetch_tensormap(&tmQ);
      int u = u_first, cur = -1, qcount = 0;
      int stage = 0;
      uint32_t round = 0;
      // L2 prefetch kPrefetch tiles ahead of the stage ring: the ring holds only kNS tiles, so
      // without it each TMA load would wait a full HBM latency behind the tile two steps back.
      int u_pf = u_first;
      long long g_pf = g_begin;
      auto prefetch_upto = [&](long long g_stop) {
        for (; g_pf < g_stop && g_pf < g_end; ++g_pf) {
          while (pre[u_pf + 1] <= g_pf) ++u_pf;
          const int s_ = (u_pf + p.u0) % p.kvp, b_ = (u_pf + p.u0) / p.kvp;
          const int pg = __ldg(p.page_table + ((size_t)s_ * p.B + b_) * p.max_pages +
                               (int)(g_pf - pre[u_pf]));
          if (pg < 0 || pg >= p.num_pages) continue;
          for (int c = 0; c < kChunks; ++c)
            tma_prefetch_l2_2d(&tmC, (4 * rank + c) * 64, pg * kPageTok);
        }
      };
      for (long long g = g_begin; g < g_end; ++g) {
        if (*(volatile int*)&tail->abort_) break;
        prefetch_upto(g + kPrefetch);
        while (pre[u + 1] <= g) ++u;
        const int s = (u + p.u0) % p.kvp, b = (u + p.u0) / p.kvp;
        if (u != cur) {  // (re)load this CTA's half of q for request b
          if (qcount > 0 && !mbar_wait(&tail->q_empty, (qcount - 1) & 1)) {
            raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
            *(volatile int*)&tail->abort_ = 1;
            break;
          }
          // the four chunks of q this CTA takes whole: 0-3 (r = 0) or 5-8 (r = 1); its half of
          // chunk 4 goes to TMEM (loaded by the softmax warps)
          mbar_arrive_expect_tx(&tail->q_full, kQBytes);
          for (int c = 0; c < kQChunks; ++c)
            tma_load_2d(q_s + c * kHeads * 128, &tmQ, (c + 5 * rank) * 64, b * kHeads,
                        &tail->q_full);
          cur = u;
          ++qcount;
        }
        // the page id is read before the wait for the stage, so its latency overlaps the wait
        const int lt = (int)(g - pre[u]);  // tile within the unit
        const int page = __ldg(p.page_table + ((size_t)s * p.B + b) * p.max_pages + lt);
        if (round > 0 && !mbar_wait(&tail->stage_empty[stage], (round - 1) & 1)) {
          raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
          *(volatile int*)&tail->abort_ = 1;
          break;
        }
        if (page < 0 || page >= p.num_pages) {
          raise_dev_error(p.err, HELIX_DEVERR_PAGE_ID);
          tail->stage_ok[stage] = 0;
          mbar_arrive(&tail->stage_full[stage]);
        } else {
          tail->stage_ok[stage] = 1;
          mbar_arrive_expect_tx(&tail->stage_full[stage], kStageBytes);
          uint8_t* st = stage_s + stage * kStageBytes;
          const int row = page * kPageTok;
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(st + c * kTok * 128, &tmC, (4 * rank + c) * 64, row,
                        &tail->stage_full[stage]);
        }
        if (++stage == kNS) { stage = 0; ++round; }
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================== score MMA issuer =======================================
    // S(i) goes out as soon as its tile has landed, its TMEM score buffer is free and its unit's
    // q is in place; the P V products have their own issuing thread (below), so a ready P V never
    // waits behind the 18 score MMAs of the next tile. Each thread's commits track only its own
    // MMAs, and the two write different accumulators.
    if (lane == 0 && active) {
      constexpr uint32_t idS = make_idesc(128, kTok, false);
      const long long n = g_end - g_begin;
      int u_s = u_first, cur = -1, qcount = 0;
      bool dead = false;
      const uint32_t qbase = smem_u32(q_s);
      for (long long ns = 0; ns < n; ++ns) {
        const long long g = g_begin + ns;
        if (*(volatile int*)&tail->abort_) break;
        while (pre[u_s + 1] <= g) ++u_s;
        if (u_s != cur) {  // this unit's q: the shared-memory chunks and the TMEM half chunk
          if (!mbar_wait(&tail->q_full, (uint32_t)(qcount & 1)) ||
              !mbar_wait(&tail->qh_full, (uint32_t)(qcount & 1))) {
            dead = true;
            break;
          }
          cur = u_s;
          ++qcount;
        }
        const int st = (int)(ns % kNS), sb = (int)(ns % kSBuf);
        if (!mbar_wait(&tail->stage_full[st], (uint32_t)((ns / kNS) & 1)) ||
            (ns >= kSBuf &&
             !mbar_wait(&tail->s_empty[sb], (uint32_t)(((ns - kSBuf) / kSBuf) & 1)))) {
          dead = true;
          break;
        }
        tc_fence_after();
        // S_partial = q[:, cols] C_tile[:, cols]^T over this CTA's 288 columns, 18 k-steps of 16
        // issued back to back. The two k-steps over the half chunk (A = q's 32 columns from TMEM)
        // go first: the tensor pipe loses time at each switch between shared-memory and
        // tensor-memory A operands, and the P V product before them also reads A from TMEM. A
        // k-step only advances the start address (16-byte units): 32 B inside a 128-byte swizzle
        // row, one chunk (q: 16 KiB, tile: 8 KiB) per 4 k-steps.
        const uint64_t a0 = smem_desc(qbase, 16, 1024, kSwizzle128);
        const uint64_t b0 = smem_desc(smem_u32(stage_s + st * kStageBytes), 16, 1024,
                                      kSwizzle128);
        const uint32_t d_s = tmem + kSCol + sb * kTok;
#pragma unroll
        for (int hj = 0; hj < 2; ++hj)  // B = this CTA's 32 columns of tile chunk 4
          tc_mma_ts(d_s, tmem + kQhCol + (uint32_t)hj * 8,
                    b0 + 4u * (1u - rank) * (kTok * 128 / 16) + 2u * ((uint32_t)hj + 2u * rank),
                    idS, hj > 0);
#pragma unroll
        for (int f = 0; f < 4 * kQChunks; ++f) {  // q's whole chunks, tile chunks r .. r + 3
          const uint32_t ch = (uint32_t)f >> 2, in_row = ((uint32_t)f & 3u) * 2u;
          tc_mma(d_s, a0 + ch * (kHeads * 128 / 16) + in_row,
                 b0 + (ch + rank) * (kTok * 128 / 16) + in_row, idS, true);
        }
        tc_commit(&tail->s_full[sb]);
        // the last tile of a unit (or of the range) releases q for the next unit
        if (g + 1 == g_end || g + 1 == pre[u_s + 1]) tc_commit(&tail->q_empty);
      }
      if (dead) {
        raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
        *(volatile int*)&tail->abort_ = 1;
      }
    }
  } else if (warp == kPvWarp) {
    // ==================================== P V issuer ==========================================
    // O += P V for each tile in order, as soon as its P is in TMEM; completing it frees the tile
    // stage (its scores were done before P existed) and the group's P buffer.
    if (lane == 0 && active) {
      constexpr uint32_t idPV = make_idesc(128, kHalfDV, true);
      const long long n = g_end - g_begin;
      int u_pv = u_first;
      bool dead = false;
      for (long long npv = 0; npv < n; ++npv) {
        if (*(volatile int*)&tail->abort_) break;
        const int pb = (int)(npv & 1);
        if (!mbar_wait(&tail->p_full[pb], (uint32_t)((npv >> 1) & 1))) {
          dead = true;
          break;
        }
        const long long g = g_begin + npv;
        while (pre[u_pv + 1] <= g) ++u_pv;
        const bool fresh = g == g_begin || g == pre[u_pv];  // first tile of a segment
        const int st = (int)(npv % kNS);
        tc_fence_after();
        const uint32_t vbase = smem_u32(stage_s + st * kStageBytes);
#pragma unroll
        for (int ks = 0; ks < kTok / 16; ++ks) {
          // A = P [128 heads x 16 tokens] from TMEM (8 columns per 16 tokens)
          // B = V [16 tokens x 256 columns], MN-major, 128-byte swizzle: 64-column groups one
          // 64-row chunk (8 KiB) apart, 8-token groups 1 KiB apart
          const uint64_t bdesc = smem_desc(vbase + ks * 16 * 128, kTok * 128, 1024, kSwizzle128);
          tc_mma_ts(tmem, tmem + kPCol + pb * (kTok / 2) + ks * 8, bdesc, idPV,
                    !(fresh && ks == 0));
        }
        tc_commit(&tail->stage_empty[st]);
        tc_commit(&tail->p_empty[pb]);
      }
      if (dead) {
        raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
        *(volatile int*)&tail->abort_ = 1;
      }
    }
  } else {
    // ================================= softmax / epilogue warps ================================
    // Two groups of four warps; group grp takes the tiles i with i % 2 == grp, so two tiles are
    // in the softmax at once. Thread h of either group owns head row h (TMEM lane h). The groups
    // share one reference maximum per row: the owner of tile i decides it from the value the
    // other group left after tile i-1 and hands it on through mpub and an mbarrier per 32-row
    // slice; each group keeps its own running sum, relative to the maximum it last saw, and the
    // two sums are merged when a segment ends. Every wait between the groups is a bounded
    // mbarrier wait: each barrier completes one phase per hand-over, and neither side can get a
    // phase ahead (the next hand-over in one direction needs the one in the other).
    const int grp = warp >> 2, slice = warp & 3;
    const int h = tid & (kHeads - 1);
    const uint32_t tl = tmem + ((uint32_t)(slice * 32) << 16);
    int n_seg = 0;  // segment ends this group has gone through
    const float sl2 = p.scale_log2;
    float m_own = -INFINITY, l_own = 0.f;  // this group's running sum and its reference maximum
    bool dead = !active;
    const uint32_t x_peer = map_peer(smem_u32(x_s), peer);
    const uint32_t xfull_peer = map_peer(smem_u32(&tail->x_full[0]), peer);
    const uint32_t xfree_peer = map_peer(smem_u32(&tail->x_free[0]), peer);
    const long long n_tiles = g_end - g_begin;
    // warp-uniform bounded waits: tcgen05.ld / st below are warp-collective
    auto wwait = [&](uint64_t* bar, uint32_t parity, bool cluster_scope) {
      if (dead) return;
      const bool ok = cluster_scope ? mbar_wait_cluster(bar, parity) : mbar_wait(bar, parity);
      if (!__all_sync(0xffffffffu, ok)) dead = true;
    };
    int u = u_first;            // unit of the tile in hand
    int len_u = 0, cur_u = -1;  // its history length (read once per unit)
    auto unit_of = [&](long long g) {
      while (pre[u + 1] <= g) ++u;
      if (u != cur_u) {
        cur_u = u;
        len_u = p.shard_lens[((u + p.u0) % p.kvp) * p.B + (u + p.u0) / p.kvp];
      }
    };
    // Segment end at a tile of the other group: hand it this group's running (m, l) (seg_ready),
    // then wait until it has read O out of TMEM (o_drained), since this group's next P V would
    // overwrite O.
    auto join_segment_end = [&]() {
      tail->seg_m[grp][h] = m_own;
      tail->seg_l[grp][h] = l_own;
      mbar_arrive(&tail->seg_ready);
      wwait(&tail->o_drained, (uint32_t)(n_seg & 1), false);
      ++n_seg;
      m_own = -INFINITY;
      l_own = 0.f;
    };
    // q's half chunk (this CTA's 32 of columns 256..319) of request bq into this thread's TMEM
    // lane: the A operand of the score k-steps over that chunk. A group loads it for the next
    // unit once it has read the scores of the unit's last tile (all of the unit's score MMAs have
    // then completed), and arrives on qh_full whether or not it could.
    auto load_q_half = [&](int bq) {
      if (!dead) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.q + ((size_t)bq * kHeads + h) * 576 + 256 + 32 * rank);
        uint32_t v[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 x = __ldg(src + c);
          v[4 * c] = x.x;
          v[4 * c + 1] = x.y;
          v[4 * c + 2] = x.z;
          v[4 * c + 3] = x.w;
        }
        tmem_st16u(tl + kQhCol, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->qh_full);
    };
    if (grp == 0 && active) load_q_half((u_first + p.u0) / p.kvp);
    float sv[kTok];
    for (long long i = grp; i < n_tiles; i += 2) {
      const long long g = g_begin + i;
      unit_of(g);
      const bool fresh = g == g_begin || g == pre[u];  // first tile of a segment
      const bool seg_end = g + 1 == g_end || g + 1 == pre[u + 1];
      const int s = (u + p.u0) % p.kvp, b = (u + p.u0) / p.kvp;
      const int lt = (int)(g - pre[u]);
      const int nvalid = min(kTok, len_u - lt * kTok);
      const int sb = (int)(i % kSBuf), st_i = (int)(i % kNS);
      // ---- A: this CTA's partial scores of tile i, from TMEM to the peer's exchange buffer ----
      dead = __any_sync(0xffffffffu, dead || *(volatile int*)&tail->abort_ != 0);
      wwait(&tail->s_full[sb], (uint32_t)((i / kSBuf) & 1), false);
      // also observe the tile's load barrier: orders the stage's validity flag and its data before
      // the zeroing of rows past the end of the history below
      wwait(&tail->stage_full[st_i], (uint32_t)((i / kNS) & 1), false);
      const bool tile_ok = tail->stage_ok[st_i] != 0;
      if (!dead) {
        tc_fence_after();
        tmem_ld64(tl + kSCol + sb * kTok, sv);
        tc_fence_before();
      } else {
#pragma unroll
        for (int c = 0; c < kTok; ++c) sv[c] = 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->s_empty[sb]);
      if (seg_end && g + 1 < g_end) {  // the next tile starts a new unit: its q half chunk
        int un = u;
        while (pre[un + 1] <= g + 1) ++un;
        load_q_half((un + p.u0) / p.kvp);
      }
      // the one exchange buffer serves the tiles in turn: tile i-1's scores must have been read
      if (i >= 1) wwait(&tail->x_free[0], (uint32_t)((i - 1) & 1), true);
      {
        const uint32_t dst = x_peer + (uint32_t)(h * 16);
#pragma unroll
        for (int c = 0; c < kTok; c += 4)
          st_async_v4(dst + (c / 4) * kHeads * 16, sv[c], sv[c + 1], sv[c + 2], sv[c + 3],
                      xfull_peer);
      }
      // the previous tile closed a segment owned by the other group: join its flush before this
      // tile's P can reach the MMA (its P V would overwrite O)
      if (fresh && i > 0) join_segment_end();
      // ---- B: add the peer's partial, softmax, P into TMEM ----
      wwait(&tail->x_full[0], (uint32_t)(i & 1), true);
      {
        const float* mine = x_s + (size_t)h * 4;
#pragma unroll
        for (int c = 0; c < kTok; c += 4) {
          const float4 v = *reinterpret_cast<const float4*>(mine + (c / 4) * kHeads * 4);
          sv[c] += v.x;
          sv[c + 1] += v.y;
          sv[c + 2] += v.z;
          sv[c + 3] += v.w;
        }
      }
      // re-arm the exchange barrier for tile i+1 (every thread of this group has observed tile i's
      // phase; the peer sends tile i+1 only after this group's hand-back below), then hand the
      // buffer back to the peer once its loads have returned
      if (h == 0 && i + 1 < n_tiles) mbar_arrive_expect_tx(&tail->x_full[0], kHeads * kTok * 4);
      keep_alive(sv);
      __syncwarp();
      if (lane == 0) remote_arrive_relaxed(xfree_peer);
      // the logit scale (times log2 e, positive) is applied inside the exponent below,
      // fma(s, sl2, -m); the row maximum is taken over the raw scores and scaled once
      if (nvalid < kTok || !tile_ok) {
#pragma unroll
        for (int c = 0; c < kTok; ++c) sv[c] = (c < nvalid && tile_ok) ? sv[c] : -INFINITY;
      }
      float mx;
      {  // tree reduction of the row maximum
        float t[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) t[c] = fmaxf(fmaxf(sv[c], sv[c + 16]), fmaxf(sv[c + 32], sv[c + 48]));
#pragma unroll
        for (int c = 0; c < 8; ++c) t[c] = fmaxf(t[c], t[c + 8]);
#pragma unroll
        for (int c = 0; c < 4; ++c) t[c] = fmaxf(t[c], t[c + 4]);
        mx = fmaxf(fmaxf(t[0], t[2]), fmaxf(t[1], t[3])) * sl2;
      }
      // V rows past the end of the history, or all of a tile whose page id is out of range (not
      // loaded: stale or never-written shared memory), are zeroed before the P V product reads
      // them, since a zero weight times a non-finite value is not zero
      const int keep = tile_ok ? nvalid : 0;
      if (keep < kTok && !dead) {
        uint8_t* stg = stage_s + st_i * kStageBytes;
        for (int e = h; e < (kTok - keep) * 4 * 8; e += kHeads) {
          const int row = keep + e / 32, rem = e % 32;
          *reinterpret_cast<uint4*>(stg + (rem / 8) * kTok * 128 + row * 128 + (rem % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      // ---- the shared reference maximum: from the other group's tile i-1, lazily raised ----
      float m_prev = -INFINITY;
      if (i > 0) {  // the other group published after tile i-1 (its ((i-1) >> 1)-th hand-over)
        wwait(&tail->m_ready[grp ^ 1][slice], (uint32_t)(((i - 1) >> 1) & 1), false);
        if (!fresh) m_prev = tail->mpub[h];
      }
      float m_new = m_prev;
      if (m_prev == -INFINITY) m_new = mx;
      else if (mx > m_prev + 8.f) m_new = mx;
      const bool rescale = m_prev != -INFINITY && m_new > m_prev;  // O holds tiles so far
      if (i + 1 < n_tiles) {
        tail->mpub[h] = m_new;
        mbar_arrive(&tail->m_ready[grp][slice]);
      }
      const float mb = m_new == -INFINITY ? 0.f : m_new;
      if (m_own != m_new) {  // this group's sum moves to the new reference
        l_own = l_own > 0.f ? l_own * fast_exp2(m_own - mb) : 0.f;
        m_own = m_new;
      }
      uint32_t pk[kTok / 2];
      float ps[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = fast_exp2(fmaf(sv[c], sl2, -mb)), p1 = fast_exp2(fmaf(sv[c + 1], sl2, -mb));
        const float p2 = fast_exp2(fmaf(sv[c + 32], sl2, -mb));
        const float p3 = fast_exp2(fmaf(sv[c + 33], sl2, -mb));
        ps[c / 2] = (p0 + p1) + (p2 + p3);
        pk[c / 2] = pack_bf16x2(p0, p1);
        pk[16 + c / 2] = pack_bf16x2(p2, p3);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) ps[c] += ps[c + 8];
#pragma unroll
      for (int c = 0; c < 4; ++c) ps[c] += ps[c + 4];
      // O is normalised by the fp32 sum (the bf16-rounded weights differ from it by < 2^-9)
      l_own += (ps[0] + ps[2]) + (ps[1] + ps[3]);
      // P(i) goes into this group's buffer, last read by PV(i-2)
      if (i >= 2) wwait(&tail->p_empty[grp], (uint32_t)(((i - 2) >> 1) & 1), false);
      if (__any_sync(0xffffffffu, rescale) && !dead) {
        // O holds tiles < i: wait for PV(i-1) (the other group's), then rescale the rows that
        // moved. PV(i+1) cannot start before P(i) is handed over, which comes after this.
        if (i >= 1) wwait(&tail->p_empty[grp ^ 1], (uint32_t)(((i - 1) >> 1) & 1), false);
        const float alpha = rescale ? fast_exp2(m_prev - m_new) : 1.f;
        tc_fence_after();
        for (int c = 0; c < kHalfDV; c += 32) {
          float o[32];
          tmem_ld32(tl + c, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(tl + c, o);
        }
        tc_fence_before();
      }
      // P row h (64 bf16) into this thread's TMEM lane: the A operand of the P V product
      if (!dead) tmem_st32u(tl + kPCol + grp * (kTok / 2), pk);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->p_full[grp]);

      if (!seg_end) continue;
      // ---- end of a segment (this group owns its last tile) ----
      wwait(&tail->seg_ready, (uint32_t)(n_seg & 1), false);  // the other group's (m, l)
      {
        // O is complete once PV(i) has finished
        wwait(&tail->p_empty[grp], (uint32_t)((i >> 1) & 1), false);
        tc_fence_after();
        const float M = m_own;  // the reference of this tile: the segment's final maximum
        const float Mb = M == -INFINITY ? 0.f : M;
        const int o_grp = grp ^ 1;
        const float m_o = tail->seg_m[o_grp][h], l_o = tail->seg_l[o_grp][h];
        const float l_run = l_own + (l_o > 0.f ? l_o * fast_exp2(m_o - Mb) : 0.f);
        const size_t orow = ((size_t)s * p.B + b) * kHeads + h;
        const bool whole = g_begin <= pre[u] && g + 1 == pre[u + 1];
        float* rec = nullptr;
        if (!whole) {
          const int slot = (g_begin >= pre[u]) ? 0 : 1;
          rec = p.seg + (((size_t)pair * 2 + slot) * 2 + rank) * kRec;
        }
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        for (int c = 0; c < kHalfDV; c += 32) {
          float o[32];
          if (!dead) tmem_ld32(tl + c, o);
          else
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0.f;
          float* dst = whole ? p.o_part + orow * kDV + rank * kHalfDV + c : rec + h * kHalfDV + c;
          const float f = whole ? inv : 1.f;
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + k) =
                make_float4(o[k] * f, o[k + 1] * f, o[k + 2] * f, o[k + 3] * f);
        }
        tc_fence_before();
        if (whole) {
          if (rank == 0) p.lse[orow] = l_run > 0.f ? (M + log2f(l_run)) * kLn2 : -INFINITY;
        } else {
          rec[kHeads * kHalfDV + h] = M;
          rec[kHeads * kHalfDV + kHeads + h] = l_run;
          rec[kHeads * kHalfDV + 2 * kHeads + h] = l_run;
          __threadfence();
          named_barrier_sync(2 + grp, kHeads);
          const int c_lo = cta_of(pre[u], W, Geff), c_hi = cta_of((long long)pre[u + 1] - 1, W, Geff);
          if (h == 0) {
            const int ticket = atomicAdd(&p.tickets[u * 2 + rank], 1);
            tail->flag = ticket == c_hi - c_lo;
          }
          named_barrier_sync(2 + grp, kHeads);
          if (tail->flag) {  // merge every cluster's segment of this unit, for this value half
            __threadfence();
            float Mm = -INFINITY;
            for (int c = c_lo; c <= c_hi; ++c) {
              const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
              Mm = fmaxf(Mm, __ldcg(p.seg + (((size_t)c * 2 + sl) * 2 + rank) * kRec +
                                    kHeads * kHalfDV + h));
            }
            const float Mmu = Mm == -INFINITY ? 0.f : Mm;
            float Lm = 0.f, LBm = 0.f;
            for (int c = c_lo; c <= c_hi; ++c) {
              const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
              const float* rc = p.seg + (((size_t)c * 2 + sl) * 2 + rank) * kRec;
              const float w_ = fast_exp2(__ldcg(rc + kHeads * kHalfDV + h) - Mmu);
              Lm += __ldcg(rc + kHeads * kHalfDV + kHeads + h) * w_;
              LBm += __ldcg(rc + kHeads * kHalfDV + 2 * kHeads + h) * w_;
            }
            const float invm = LBm > 0.f ? 1.f / LBm : 0.f;
            for (int cc = 0; cc < kHalfDV; cc += 4) {
              float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
              for (int c = c_lo; c <= c_hi; ++c) {
                const int sl = (range_begin(c, W, Geff) >= pre[u]) ? 0 : 1;
                const float* rc = p.seg + (((size_t)c * 2 + sl) * 2 + rank) * kRec;
                const float w_ = fast_exp2(__ldcg(rc + kHeads * kHalfDV + h) - Mmu);
                const float4 v = __ldcg(reinterpret_cast<const float4*>(rc + h * kHalfDV + cc));
                acc.x += v.x * w_;
                acc.y += v.y * w_;
                acc.z += v.z * w_;
                acc.w += v.w * w_;
              }
              *reinterpret_cast<float4*>(p.o_part + orow * kDV + rank * kHalfDV + cc) =
                  make_float4(acc.x * invm, acc.y * invm, acc.z * invm, acc.w * invm);
            }
            if (rank == 0) p.lse[orow] = Lm > 0.f ? (Mm + log2f(Lm)) * kLn2 : -INFINITY;
            named_barrier_sync(2 + grp, kHeads);
            if (h == 0) p.tickets[u * 2 + rank] = 0;
          }
        }
      }
      mbar_arrive(&tail->o_drained);
      ++n_seg;
      m_own = -INFINITY;
      l_own = 0.f;
    }
    // the range's last tile belongs to the other group: join its flush
    if (n_tiles > 0 && ((n_tiles - 1) & 1) != grp) join_segment_end();
  }

  // ---- teardown: every thread of both CTAs gets here (all waits above are bounded) ----
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote store or arrival can target this CTA after this point
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

size_t mla_partial_smem_bytes(int units) { return kSmemFixed + (size_t)(units + 1) * sizeof(int); }
size_t mla_segment_record_floats() { return kRec; }

helix_status mla_partial_launch(const CUtensorMap& tmC, const CUtensorMap& tmQ,
                                const MlaParams& p, int grid, cudaStream_t stream) {
  const size_t smem = mla_partial_smem_bytes(p.units);
  if (allow_max_dynamic_smem(reinterpret_cast<const void*>(mla_partial_kernel)) != cudaSuccess)
    return HELIX_ERR_CUDA;
  mla_partial_kernel<<<grid, kThreads, smem, stream>>>(tmC, tmQ, p);
  return cudaGetLastError() == cudaSuccess ? HELIX_OK : HELIX_ERR_CUDA;
}

}  // namespace helix
