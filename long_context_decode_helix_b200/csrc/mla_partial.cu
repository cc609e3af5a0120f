// mla_partial.cu -- per-shard partial decode attention for absorbed multi-head latent attention
// (MLA) on the 5th-generation tensor cores, as pair-wide (two-SM) MMAs with accumulators in tensor
// memory.
//
// What it computes: 128 query heads attend to ONE shared latent KV head (the paper summary's
// tensor-parallelism paragraph notes that MLA "effectively" has one KV head, which is why its KV
// cannot be split by heads and KV parallelism is needed). With the absorbed formulation the latent
// row c_t (576 wide) is the key and its first 512 columns are the value:
//     z_{h,t} = scale * <q_h, c_t>,  O_s[h] = sum_t e^{z - m} c_t[0:512] / sum_t e^{z - m},
//     lse_s[h] = m + ln sum_t e^{z - m}
// over the tokens T_s of KVP shard s (paper summary, paragraph on KV parallelism).
//
// Sizes force two SMs per tile. O for 128 heads x 512 columns in fp32 fills all 512 TMEM columns
// of one SM, and q (128 x 576 bf16) alone is 144 KiB. A cluster of two CTAs therefore splits the
// HEADS: CTA r owns heads [64 r, 64 r + 64), holds their q (72 KiB) in shared memory and their O
// (64 x 512 fp32) in 256 TMEM columns, and every MMA is a pair-wide tcgen05.mma.cta_group::2
// issued by a thread of CTA 0, in which each SM computes the rows of its own heads:
//   * scores S = q C^T per 128-token tile (two pages; CTA r loads page r of the two), M = 128
//     heads (64 per SM), N = 128 tokens (each CTA supplies the 64 rows of its page as its half of
//     B), K = 576 in 36 steps: each SM ends with the complete scores of its 64 heads for all 128
//     tokens, so the softmax needs nothing from the other SM;
//   * O += P V per tile, M = 128 heads (64 per SM), N = 256 value columns per MMA (each CTA
//     supplies 128 of them: CTA r the 64-column chunks 2r, 2r + 1 of each 256-column block), K =
//     128 tokens. P is written to shared memory by the softmax warps (the A operand, K-major);
//     V is read again from L2 into the value ring (MN-major), two 64-column chunks x 64 tokens.
// Operands stream through two rings of 16 KiB shared-memory slots, one per operand, each filled by
// a producer warp in both CTAs: the score ring (3 slots) takes this CTA's page of each tile as five
// slots of two 64-column chunks (one 3-D TMA box each; the fifth holds chunk 8 and zeros), the
// value ring (4 slots, a whole tile) takes, per column block j and page, this CTA's two 64-column
// chunks of that page (read again, from L2). Every TMA load of either CTA completes on CTA 0's barrier of its slot; the MMAs'
// commits reach both CTAs (tcgen05.commit multicast). No TMA load uses cluster multicast.
//
// Issue: a thread issuing a pair-wide tcgen05.mma is busy for longer than the tensor pipe needs
// for these shapes, so three threads of CTA 0 issue: two take the first / second half of the
// k-steps of every chunk into two score accumulators (the softmax adds them), the third issues
// P V. Warps 4-11 are the softmax / epilogue warps.
// TMEM lane l holds head l's scores of the first page of the tile for l < 64, and lane 64 + l the
// same head's scores of the second page (the two-SM layout of an M = 64-per-SM accumulator). Two
// softmax threads read each lane, 32 columns each, once: the score buffer is released as soon as
// that read completes, and the four threads of a head combine their row maxima through shared
// memory. The tensor pipe computes the scores of tile i + 1 while the softmax works on tile i;
// the scores and P each have two buffers. The reference maximum moves lazily (only when a row
// maximum exceeds it by more than 8 in base-2 units), so weights stay below 2^8 and the TMEM
// rescale of O is rare; the logit scale is applied inside the exponent.
// Work is split over the (request, shard) units as in the GQA kernels: each cluster takes an equal
// contiguous range of 128-token tiles; split units are merged by the last arriving cluster, per
// CTA (its 64 heads).
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
constexpr int kHc = 64;                  // heads per CTA
constexpr int kD = 576, kDV = 512;
constexpr int kPage = 64;                // tokens per page (and per CTA per tile)
constexpr int kTile = 2 * kPage;         // tokens per tile of the pair
constexpr int kChunks = 9;               // 64-column chunks of a latent row
constexpr int kSlot = 8192;              // one 64-column chunk of a page (64 rows x 128 B)
constexpr int kQSlot = 2 * kSlot;        // score ring slot: two chunks of a page
constexpr int kRingQ = 3;                // score-operand ring slots
constexpr int kQSlotsPerTile = 5;        // chunks (0,1) (2,3) (4,5) (6,7) (8,-)
constexpr int kVSlot = 2 * kSlot;        // value ring slot: 128 value columns of one page
constexpr int kRingV = 4;                // value-operand ring slots (a whole tile: the fourth slot
                                         // of a tile would otherwise load only after P V took the first)
constexpr int kQBytes = kChunks * kHc * 128;  // 72 KiB
constexpr int kPBytes = 2 * kHc * 128;        // one tile's P: two 64-token K-chunks, 16 KiB
constexpr uint32_t kOCol = 0, kSCol = 256, kTmemCols = 512;
// Warp roles: the two score issuers, the P V issuer and the value producer on warps 0-3, the score
// producer on warp 12, the softmax warps on 4-11 (warp w reads TMEM lanes 32 (w % 4) .. + 31; warps
// w and w + 4 take the two 32-column halves of those lanes' scores).
constexpr int kMmaWarp2 = 0, kMmaWarp = 1, kPvWarp = 2, kValueWarp = 3, kSoftmaxWarp0 = 4,
              kSoftmaxWarps = 8, kProducerWarp = 12;
constexpr int kSoftThreads = kSoftmaxWarps * 32;
constexpr int kThreads = 13 * 32;
// two softmax warps per TMEM lane quarter, one per 32-column half of the page's scores
static_assert(kSoftmaxWarps == 8 && kProducerWarp == kSoftmaxWarp0 + kSoftmaxWarps &&
                  kThreads == (kProducerWarp + 1) * 32,
              "the softmax's column split is written for two warps per lane quarter");
constexpr int kRec = kHc * (kDV + 3);    // floats per segment record (this CTA's heads)
constexpr float kLazy = 8.f;             // base-2 headroom before the reference maximum moves
constexpr int kPf = 2;                   // tiles whose pages are fetched into L2 ahead of the ring
constexpr int kPid = 8;                  // page-id queue of the producer (tiles)

struct MlaTail {
  uint64_t full_q[kRingQ];   // CTA 0: its producer's arrival and both CTAs' TMA bytes
  uint64_t empty_q[kRingQ];  // both: the MMAs that read the slot are done
  uint64_t full_v[kRingV];   // the same for the value ring
  uint64_t empty_v[kRingV];
  uint64_t s_full[2];      // both: the scores of a tile are in TMEM (both score issuers)
  uint64_t s_empty[2];     // CTA 0: the 8 softmax warps of each CTA read them
  uint64_t p_full[2];      // CTA 0: the 8 softmax warps of each CTA wrote P (and rescaled O)
  uint64_t p_empty[2];     // both: P V of the tile is done
  uint64_t q_full;         // CTA 0: its producer's arrival and both CTAs' q bytes
  uint64_t q_empty;        // both: the last score MMAs of a unit (both issuers) are done
  uint64_t mma_done;       // both: every MMA issued by the three issuers has completed
  // [tile parity][lane][column half]: row maxima of a quarter tile (read as 8-byte pairs)
  alignas(8) float xmax[2][kHeads][2];
  float xl[2][kHeads];       // [column half][lane]: row sums of a quarter at a segment end
  int pid[kPid][2];        // producer only: page ids (or -1) of the two pages of a tile
  uint32_t tmem_base;
  int flag;
  int abort_;
};

constexpr size_t kSmemFixed =
    1024 + kQBytes + 2 * kPBytes + (size_t)kRingQ * kQSlot + (size_t)kRingV * kVSlot +
    sizeof(MlaTail);

// ------------------------------------------------------------------------------------------------
// cluster, mbarrier and tcgen05 helpers

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
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrival on a barrier of either CTA (shared::cluster address) that orders this thread's earlier
// shared-memory writes for the reader (release, CTA scope: the form the pair's pipelines use).
__device__ __forceinline__ void arrive_remote(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Arrival that orders nothing (the data it announces was consumed, not produced).
__device__ __forceinline__ void arrive_remote_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar)
               : "memory");
}
// Counts `tx` bytes as arrived on a barrier of either CTA without an arrival (for data written by
// the threads themselves instead of TMA; the caller orders those writes first).
__device__ __forceinline__ void complete_tx_remote(uint32_t bar, uint32_t tx) {
  asm volatile("mbarrier.complete_tx.relaxed.cluster.shared::cluster.b64 [%0], %1;" ::"r"(bar),
               "r"(tx)
               : "memory");
}
// bounded wait on one of this CTA's barriers (phases completed by TMA bytes, the MMA's commits or
// arrivals from either CTA)
__device__ __forceinline__ bool mbar_wait_pair(uint64_t* bar, uint32_t parity) {
  return mbar_wait(bar, parity);
}
// 2-D TMA tile load into this CTA's shared memory whose completion (bytes) is counted on a barrier
// of either CTA of the pair (given by its shared::cluster address). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, int32_t x,
                                                 int32_t y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

// The same for a 3-D box (the latent pool seen as [chunk][row][64 columns]).
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, int32_t x,
                                                 int32_t y, int32_t z, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
      : "memory");
}
// Brings `bytes` (a multiple of 16) of global memory at a 16-byte aligned address into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// arrive on the same barrier of both CTAs once every pair-wide MMA issued so far has completed
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// pair-wide D (+)= A B, both operands in shared memory (each CTA supplies its half of A by rows and
// of B by columns, at the same shared-memory offsets)
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane; the registers are valid after
// tmem_wait_ld()
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float (&v)[32]) {
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
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Two IEEE fp32 additions / fused multiply-adds (round to nearest) in one instruction.
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%0, %1};\n mov.b64 rb, {%2, %3};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}
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
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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
// 16-byte units, descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor for kind::f16: fp32 accumulate, bf16 A and B, A K-major, B K-major or
// MN-major; M is the pair-wide M.
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

// The unit that tile g of the cluster's range belongs to, with the unit's first tile, the first
// tile past it, its shard row (s * B + b) and its token count kept in registers: they are read
// from shared memory only when the unit changes.
struct UnitCursor {
  int u, first, next, row, len;
  __device__ __forceinline__ void start(const int* pre, const int* urow, const int* ulen, int u0) {
    u = u0;
    first = pre[u];
    next = pre[u + 1];
    row = urow[u];
    len = ulen[u];
  }
  // moves to the unit of tile g (g never decreases); true when the unit changed
  template <class G>
  __device__ __forceinline__ bool seek(const int* pre, const int* urow, const int* ulen, G g) {
    if (g < next) return false;
    do {
      ++u;
      first = next;
      next = pre[u + 1];
    } while (next <= g);
    row = urow[u];
    len = ulen[u];
    return true;
  }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_partial_kernel(const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmQ, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* q_s = smem;                      // [9 chunks][64 rows][128 B]
  uint8_t* p_s = q_s + kQBytes;             // [2 groups][2 token chunks][64 rows][128 B]
  uint8_t* ring_q = p_s + 2 * kPBytes;      // [kRingQ][2 chunks][64 rows][128 B]: score operand
  uint8_t* ring_v = ring_q + (size_t)kRingQ * kQSlot;  // [kRingV][2 chunks][64 rows][128 B]
  MlaTail* tail = reinterpret_cast<MlaTail*>(ring_v + (size_t)kRingV * kVSlot);
  int* pre = reinterpret_cast<int*>(tail + 1);  // [U + 1]: first tile of each unit
  int* urow = pre + (p.units + 1);               // [U]: s * B + b, the unit's shard_lens index
  int* ulen = urow + p.units;                    // [U]: the unit's token count (capped)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int U = p.units;

  // ---- 128-token tiles per unit and their prefix sums ----
  for (int u = tid; u < U; u += kThreads) {
    const int s = (u + p.u0) % p.kvp, b = (u + p.u0) / p.kvp;
    int len = p.shard_lens[s * p.B + b];
    if (len > p.max_pages * kPage) {
      if (blockIdx.x == 0) raise_dev_error(p.err, HELIX_DEVERR_CAPACITY);
      len = p.max_pages * kPage;
    }
    pre[u + 1] = len > 0 ? (len + kTile - 1) / kTile : 0;
    urow[u] = s * p.B + b;
    ulen[u] = max(len, 0);
  }
  if (tid == 0) {
    pre[0] = 0;
    for (int i = 0; i < kRingQ; ++i) {
      mbar_init(&tail->full_q[i], 1);   // CTA 0's producer, with both CTAs' bytes
      mbar_init(&tail->empty_q[i], 2);  // the commits of both score issuers
    }
    for (int i = 0; i < kRingV; ++i) {
      mbar_init(&tail->full_v[i], 1);
      mbar_init(&tail->empty_v[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tail->s_full[i], 2);  // the commits of both score issuers
      mbar_init(&tail->s_empty[i], 2 * kSoftmaxWarps);  // the softmax warps of both CTAs
      mbar_init(&tail->p_full[i], 2 * kSoftmaxWarps);
      mbar_init(&tail->p_empty[i], 1);
    }
    mbar_init(&tail->q_full, 1);
    mbar_init(&tail->q_empty, 2);
    mbar_init(&tail->mma_done, 3);  // the three issuing threads' final commits
    tail->flag = 0;
    tail->abort_ = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {  // all 512 TMEM columns of both SMs, allocated by the pair together
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&tail->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
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
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrival

  const uint32_t tmem = tail->tmem_base;
  const long long W = pre[U];
  // units with no tokens: O_s = 0, lse_s = -inf (this CTA's heads)
  for (int u = pair; u < U; u += npairs) {
    if (pre[u + 1] != pre[u]) continue;
    const size_t row0 = (size_t)urow[u] * kHeads + (size_t)rank * kHc;
    for (int i = tid; i < kHc * kDV; i += kThreads) p.o_part[row0 * kDV + i] = 0.f;
    for (int i = tid; i < kHc; i += kThreads) p.lse[row0 + i] = -INFINITY;
  }
  const int Geff = (int)min((long long)npairs, W);
  const bool active = pair < Geff;
  const long long g_begin = active ? range_begin(pair, W, Geff) : 0;
  const long long g_end = active ? range_begin(pair + 1, W, Geff) : 0;
  const long long n_tiles = g_end - g_begin;
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
  const uint32_t lead_full_q0 = map_rank(&tail->full_q[0], 0);
  const uint32_t lead_full_v0 = map_rank(&tail->full_v[0], 0);
  const uint32_t lead_q_full = map_rank(&tail->q_full, 0);
  const int oob_row = p.num_pages * kPage;  // a row past the pool: TMA fills a box there with 0

  // One ring of slots, walked in order by one producer warp (both CTAs) and one issuing thread
  // (CTA 0): the producer takes a slot once the MMAs of its previous fill are done.
  struct Ring {
    uint64_t* full;
    uint64_t* empty;
    int n;
    int k = 0;
    uint32_t round = 0;
  };
  // producer side: the next slot, waited for warp-wide (bounded); returns -1 when a wait ran out
  auto acquire = [&](Ring& r) -> int {
    const int k = r.k;
    if (r.round > 0) {
      const bool ok = mbar_wait_pair(&r.empty[k], (r.round - 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) return -1;
    }
    if (++r.k == r.n) {
      r.k = 0;
      ++r.round;
    }
    return k;
  };
  // issuer side: the next slot once both CTAs' data for it has landed; -1 when the wait ran out
  auto take = [&](Ring& r) -> int {
    const int k = r.k;
    if (!mbar_wait_pair(&r.full[k], r.round & 1)) return -1;
    if (++r.k == r.n) {
      r.k = 0;
      ++r.round;
    }
    return k;
  };

  if (warp == kProducerWarp) {
    // ============================ score-operand producer (both CTAs) =============================
    // For each tile, this CTA's page in five slots of two 64-column chunks (one 3-D TMA each; the
    // fifth holds chunk 8 and zeros); q of a new unit's request. Page ids are used kPf tiles ahead
    // (lanes 0 and 1 take the tile's two pages) to bring this CTA's page into L2, so the ring's
    // loads find it there; their global loads are issued one tile before they are needed.
    if (active) {
      if (lane == 0) {
        prefetch_tensormap(&tmC);
        prefetch_tensormap(&tmQ);
      }
      Ring rq{tail->full_q, tail->empty_q, kRingQ};
      bool dead = false;
      UnitCursor at_r;
      at_r.start(pre, urow, ulen, u_first);
      int r_raw = -1, r_len = 0, r_lp = 0;  // loads in flight for the next tile to resolve
      auto issue_ids = [&](long long t) {  // starts the loads of tile t's page ids (no wait)
        const long long g = g_begin + t;
        at_r.seek(pre, urow, ulen, g);
        r_lp = 2 * (int)(g - at_r.first) + (lane & 1);
        r_len = at_r.len;
        r_raw = r_lp < p.max_pages ? __ldg(p.page_table + (size_t)at_r.row * p.max_pages + r_lp)
                                   : -1;
      };
      auto finish_ids = [&](long long t) {  // page ids of tile t into the queue; L2 prefetch
        int pg = -1;
        if (r_lp * kPage < r_len) {
          if (r_raw < 0 || r_raw >= p.num_pages) {
            if (lane < 2) raise_dev_error(p.err, HELIX_DEVERR_PAGE_ID);
          } else {
            pg = r_raw;
          }
        }
        if (lane < 2) tail->pid[t % kPid][lane] = pg;
        const int mine = __shfl_sync(0xffffffffu, pg, (int)rank);
        if (lane == 0 && mine >= 0)
          bulk_prefetch_l2(p.pool + (size_t)mine * kPage * (kD * 2), kPage * kD * 2);
        __syncwarp();
      };
      UnitCursor at_q;
      at_q.start(pre, urow, ulen, u_first);
      int cur = -1, qcount = 0;
      for (long long t = 0; t < kPf && t < n_tiles; ++t) {
        issue_ids(t);
        finish_ids(t);
      }
      if (kPf < n_tiles) issue_ids(kPf);
      for (long long i = 0; i < n_tiles && !dead; ++i) {
        if ((i & 7) == 0 && *(volatile int*)&tail->abort_) { dead = true; break; }
        if (i + kPf < n_tiles) {
          finish_ids(i + kPf);
          if (i + kPf + 1 < n_tiles) issue_ids(i + kPf + 1);
        }
        const long long g = g_begin + i;
        at_q.seek(pre, urow, ulen, g);
        const int u = at_q.u;
        if (u != cur) {  // this CTA's 64 heads of q for the unit's request, once the previous
                         // unit's score MMAs are done with the buffer. It goes before the tile's
                         // chunks: the issuers take no chunk of the unit before q, and the ring is
                         // shorter than a tile.
          if (qcount > 0) {
            const bool ok = mbar_wait_pair(&tail->q_empty, (qcount - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
          }
          if (lane == 0) {
            const int b = at_q.row % p.B;
            if (rank == 0) mbar_arrive_expect_tx(&tail->q_full, 2 * kQBytes);
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d_pair(q_s + c * kHc * 128, &tmQ, 64 * c, b * kHeads + (int)rank * kHc,
                               lead_q_full);
          }
          cur = u;
          ++qcount;
        }
        const int pg = tail->pid[i % kPid][rank];
        const int y = pg < 0 ? oob_row : pg * kPage;
        for (int sl = 0; sl < kQSlotsPerTile; ++sl) {
          const int k = acquire(rq);
          if (k < 0) { dead = true; break; }
          if (lane == 0) {
            if (rank == 0) mbar_arrive_expect_tx(&tail->full_q[k], 2 * kQSlot);
            tma_load_3d_pair(ring_q + (size_t)k * kQSlot, &tmC, 0, y, 2 * sl, lead_full_q0 + 8u * k);
          }
        }
      }
      if (dead && lane == 0) {
        raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
        *(volatile int*)&tail->abort_ = 1;
      }
    }
  } else if (warp == kValueWarp) {
    // ============================ value-operand producer (both CTAs) =============================
    // For each tile, column block j and page `half` of the tile: this CTA's two 64-column chunks
    // (4 j + 2 rank, + 1) of the page's 64 tokens, read again (from L2: both pages of the tile were
    // just loaded for the scores). The next tile's page ids are read while this tile's slots fill.
    if (active) {
      if (lane == 0) prefetch_tensormap(&tmC);
      Ring rv{tail->full_v, tail->empty_v, kRingV};
      bool dead = false;
      UnitCursor at, at_n;
      at.start(pre, urow, ulen, u_first);
      at_n = at;
      auto ids = [&](long long t) -> int {  // lane 0: page A, lane 1: page B of tile t
        const long long g = g_begin + t;
        at_n.seek(pre, urow, ulen, g);
        const int lp = 2 * (int)(g - at_n.first) + lane;
        if (lane >= 2 || lp * kPage >= at_n.len) return -1;
        const int pg = __ldg(p.page_table + (size_t)at_n.row * p.max_pages + lp);
        return (pg < 0 || pg >= p.num_pages) ? -1 : pg;
      };
      int nxt = n_tiles > 0 ? ids(0) : -1;
      for (long long t = 0; t < n_tiles && !dead; ++t) {
        if ((t & 7) == 0 && *(volatile int*)&tail->abort_) { dead = true; break; }
        const int pgA = __shfl_sync(0xffffffffu, nxt, 0), pgB = __shfl_sync(0xffffffffu, nxt, 1);
        if (t + 1 < n_tiles) nxt = ids(t + 1);
        const long long g = g_begin + t;
        at.seek(pre, urow, ulen, g);
        const int tt = (int)(g - at.first), len = at.len;
        for (int j = 0; j < 2 && !dead; ++j) {
          for (int half = 0; half < 2; ++half) {
            const int k = acquire(rv);
            if (k < 0) { dead = true; break; }
            const int pg = half ? pgB : pgA;
            const int nvalid = min(max(len - (2 * tt + half) * kPage, 0), kPage);
            uint8_t* slot = ring_v + (size_t)k * kVSlot;
            const int cb = 4 * j + 2 * (int)rank;
            // CTA 0 expects both CTAs' bytes of the slot
            if (lane == 0 && rank == 0) mbar_arrive_expect_tx(&tail->full_v[k], 2 * kVSlot);
            if (pg < 0 || nvalid == 0 || nvalid == kPage) {
              // the whole page, or nothing of the history (zeros from past the pool)
              if (lane == 0) {
                const int y = (pg < 0 || nvalid == 0) ? oob_row : pg * kPage;
                tma_load_3d_pair(slot, &tmC, 0, y, cb, lead_full_v0 + 8u * k);
              }
            } else {
              // the last, partial page of a shard: rows of the history are copied, rows past it
              // are zeroed (a zero weight times a non-finite stale value would not be zero), in
              // the 128-byte swizzled layout TMA writes
              for (int e = lane; e < 2 * kPage * 8; e += 32) {
                const int sb = e >> 9, r = (e >> 3) & (kPage - 1), un = e & 7;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (r < nvalid)
                  v = __ldg(reinterpret_cast<const uint4*>(
                      p.pool + ((size_t)pg * kPage + r) * (kD * 2) + (64 * (cb + sb) + 8 * un) * 2));
                *reinterpret_cast<uint4*>(slot + sb * kSlot + r * 128 + ((un ^ (r & 7)) << 4)) = v;
              }
              fence_proxy_async_smem();  // the generic-proxy stores before the MMA's reads
              __syncwarp();
              if (lane == 0) {
                asm volatile("fence.acq_rel.cluster;" ::: "memory");
                complete_tx_remote(lead_full_v0 + 8u * k, kVSlot);
              }
            }
          }
        }
      }
      if (dead && lane == 0) {
        raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
        *(volatile int*)&tail->abort_ = 1;
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp2 || warp == kPvWarp) {
    // ====================== MMA issuers (CTA 0: one thread in each of three warps) ===============
    // Issuing a pair-wide tcgen05.mma occupies its thread for longer than the tensor pipe needs to
    // execute one of these shapes (64 x 128 x 16 and 64 x 256 x 16 per SM), so one thread cannot
    // keep the pipe busy. Three threads on three SM sub-partitions issue: score issuer `role` 0 / 1
    // takes the first / second half of the k-steps of every 64-column chunk into its own score
    // accumulator (the softmax adds the two), the third issues P V. Descriptors are formed once and advanced by
    // constants, so little but the MMAs themselves runs between them.
    const int role = warp == kMmaWarp ? 0 : warp == kMmaWarp2 ? 1 : 2;
    if (rank == 0 && lane == 0 && active) {
      constexpr uint32_t idQK = make_idesc(128, kTile, false);
      constexpr uint32_t idPV = make_idesc(128, 256, true);
      bool dead = false;
      UnitCursor at;
      at.start(pre, urow, ulen, u_first);
      if (role < 2) {
        // S_role(i) = the k-steps kk = 2 role, 2 role + 1 of every 64-column chunk c of tile i:
        // sum of q[:, 64c + 16kk : +16] C[:, 64c + 16kk : +16]^T. Both threads wait for every
        // slot in ring order (a thread that skipped slots could mistake an old phase of a slot for
        // the one it wants: the waits go by phase parity) and each commits the slot's release
        // (count 2). Slot sl of tile i is ring position 5 i + sl; a k-step of 16 columns advances
        // the start address 32 B (2 descriptor units) inside the 128-byte swizzled rows; chunk
        // c + 1 of a slot follows chunk c at 8 KiB.
        const uint64_t qd = smem_desc(smem_u32(q_s), 16, 1024) + (uint64_t)(4 * role);
        const uint64_t rd = smem_desc(smem_u32(ring_q), 16, 1024) + (uint64_t)(4 * role);
        int cur = -1, qcount = 0;
        uint32_t pos = 0;  // ring position of the next slot
        for (long long i = 0; i < n_tiles && !dead; ++i) {
          if ((i & 7) == 0 && *(volatile int*)&tail->abort_) { dead = true; break; }
          const long long g = g_begin + i;
          at.seek(pre, urow, ulen, g);
          if (at.u != cur) {
            if (!mbar_wait_pair(&tail->q_full, (uint32_t)(qcount & 1))) { dead = true; break; }
            cur = at.u;
            ++qcount;
          }
          if (i >= 2) {
            if (!mbar_wait_pair(&tail->s_empty[i & 1], (uint32_t)(((i - 2) >> 1) & 1))) {
              dead = true;
              break;
            }
            tc_fence_after();  // the softmax's TMEM reads of the buffer came first
          }
          const uint32_t d_s = tmem + kSCol + (uint32_t)(i & 1) * kTile + (uint32_t)role * (kTile / 2);
          for (int sl = 0; sl < kQSlotsPerTile; ++sl, ++pos) {
            const int ks = (int)(pos % kRingQ);
            if (!mbar_wait_pair(&tail->full_q[ks], (uint32_t)((pos / kRingQ) & 1))) {
              dead = true;
              break;
            }
            const uint64_t bs = rd + (uint64_t)((ks * kQSlot) >> 4);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int c = 2 * sl + cc;
              if (c >= kChunks) break;
              const uint64_t a = qd + (uint64_t)((c * (kHc * 128)) >> 4);
              const uint64_t bd = bs + (uint64_t)((cc * kSlot) >> 4);
              tc_mma_pair(d_s, a, bd, idQK, c != 0);
              tc_mma_pair(d_s, a + 2, bd + 2, idQK, true);
            }
            tc_commit_pair(&tail->empty_q[ks]);
          }
          if (dead) break;
          tc_commit_pair(&tail->s_full[i & 1]);
          // the last tile of a unit (or of the range) releases q for the next unit
          if (g + 1 == g_end || g + 1 == at.next) tc_commit_pair(&tail->q_empty);
        }
      } else {
        // O[:, 256 j : 256 j + 256] += P V per page `half` of the tile: 4 k-steps of 16 tokens.
        // A = P of this CTA's 64 heads (K-major, page `half` is a 64-token chunk, 32 B per step);
        // B = V slot (MN-major: two 64-column sub-blocks 8 KiB apart, 8-token groups 1 KiB apart,
        // 16 tokens = 2 KiB per step).
        const uint64_t pd = smem_desc(smem_u32(p_s), 16, 1024);
        const uint64_t vd = smem_desc(smem_u32(ring_v), kSlot, 1024);
        Ring rv{tail->full_v, tail->empty_v, kRingV};
        for (long long t = 0; t < n_tiles && !dead; ++t) {  // O += P V of tile t
          if ((t & 7) == 0 && *(volatile int*)&tail->abort_) { dead = true; break; }
          if (!mbar_wait_pair(&tail->p_full[t & 1], (uint32_t)((t >> 1) & 1))) {
            dead = true;
            break;
          }
          tc_fence_after();  // P (generic stores, proxy-fenced) and the O rescale came first
          const long long g = g_begin + t;
          at.seek(pre, urow, ulen, g);
          const bool fresh = t == 0 || g == at.first;  // first tile of a segment
          const uint64_t pt = pd + (uint64_t)(((uint32_t)(t & 1) * kPBytes) >> 4);
          for (int j = 0; j < 2 && !dead; ++j) {
            for (int half = 0; half < 2; ++half) {
              const int ks = take(rv);
              if (ks < 0) { dead = true; break; }
              const uint64_t a = pt + (uint64_t)((half * (kHc * 128)) >> 4);
              const uint64_t bd = vd + (uint64_t)((ks * kVSlot) >> 4);
#pragma unroll
              for (int kt = 0; kt < 4; ++kt)
                tc_mma_pair(tmem + kOCol + (uint32_t)j * 128, a + 2 * kt, bd + 128 * kt, idPV,
                            !(fresh && half == 0 && kt == 0));
              tc_commit_pair(&tail->empty_v[ks]);
            }
          }
          if (dead) break;
          tc_commit_pair(&tail->p_empty[t & 1]);
        }
      }
      if (dead) {
        raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
        *(volatile int*)&tail->abort_ = 1;
      }
    }
    // every MMA this thread issued (none on CTA 1) completes before the teardown
    if (rank == 0 && lane == 0) tc_commit_pair(&tail->mma_done);
  } else {
    // ============================== softmax / epilogue warps =====================================
    // Thread (lr, ch) reads TMEM lane lr: local head hl = lr % 64, page half = lr / 64 of each tile,
    // and of that page's 64 tokens the 32 in column half ch = 32 ch .. 32 ch + 31. The four threads
    // of a head (two halves x two column halves) agree on its maximum through shared memory; those
    // four warps have the same parity, so each tile's exchange waits on named barrier 1 (even warps)
    // or 2 (odd warps), and only a segment end, where all eight meet, on barrier 3.
    const int ch = (warp - kSoftmaxWarp0) >> 2;  // column half of the scores this warp reads
    const int lr = 32 * (warp & 3) + lane;       // TMEM lane of this thread
    const int hl = lr & (kHc - 1);      // local head (row of this CTA's q)
    const int half = lr >> 6;           // which page of the tile this lane's scores belong to
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t lead_s_empty = map_rank(&tail->s_empty[0], 0);
    const uint32_t lead_p_full = map_rank(&tail->p_full[0], 0);
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY;  // the head's reference maximum (base-2 logits), shared by its threads
    float l_own = 0.f;        // running sum of this thread's weights relative to m_ref
    bool dead = !active;
    auto wwait = [&](uint64_t* bar, uint32_t parity) {  // warp-uniform bounded wait
      if (dead) return;
      if (!__all_sync(0xffffffffu, mbar_wait_pair(bar, parity))) dead = true;
    };
    UnitCursor at, at_n;
    at.start(pre, urow, ulen, u_first);
    at_n = at;
    // This lane's page id of tile i + 1 is loaded while tile i is worked on (a page-table line is
    // often no longer in L2 by the time it is needed).
    int nx_raw = -1;
    // tile indices fit in 32 bits (a launch's tiles are counted in int)
    const int gb = (int)g_begin, ge = (int)g_end, nt = (int)n_tiles;
    const int* pt_row = p.page_table + (size_t)at_n.row * p.max_pages;  // at_n's page-table row
    auto load_next = [&](int t) {
      const int g = gb + t;
      if (at_n.seek(pre, urow, ulen, g)) pt_row = p.page_table + (size_t)at_n.row * p.max_pages;
      const int lp = 2 * (g - at_n.first) + half;
      nx_raw = lp < p.max_pages ? __ldg(pt_row + lp) : -1;
    };
    if (nt > 0) load_next(0);
    for (int i = 0; i < nt; ++i) {
      const int g = gb + i;
      at.seek(pre, urow, ulen, g);
      const int u = at.u;
      const int len_u = at.len, raw = nx_raw;  // raw: loaded during the previous tile
      if (i + 1 < nt) load_next(i + 1);
      const bool fresh = g == gb || g == at.first;
      const bool seg_end = g + 1 == ge || g + 1 == at.next;
      const int tt = g - at.first;
      const int nvalid = min(max(len_u - (2 * tt + half) * kPage, 0), kPage);
      const bool page_ok = nvalid > 0 && raw >= 0 && raw < p.num_pages;
      const int sb = (int)(i & 1);
      if (fresh) {  // a new segment: O starts over (its first P V overwrites the accumulator)
        m_ref = -INFINITY;
        l_own = 0.f;
      }
      // ---- this thread's 32 scores of tile i: S = S_0 + S_1 (the two score issuers' accumulators,
      // 64 columns each), read once; the buffer is released as soon as the read has completed ----
      dead = __any_sync(0xffffffffu, dead || ((i & 7) == 0 && *(volatile int*)&tail->abort_ != 0));
      wwait(&tail->s_full[sb], (uint32_t)((i >> 1) & 1));
      const uint32_t sa = tl + kSCol + (uint32_t)sb * kTile + 32u * (uint32_t)ch;
      const bool keep_all = nvalid == kPage && page_ok;
      float x[32];
      float mx = -INFINITY;
      if (!dead) {
        tc_fence_after();
        float v1[32];
        tmem_ld32_nowait(sa, x);
        tmem_ld32_nowait(sa + kTile / 2, v1);
        tmem_wait_ld();
        float t[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) t[c] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; c += 2) add2(x[c], x[c + 1], v1[c], v1[c + 1]);
        // rare: the last, partial page of a shard, or a page id out of range
        if (__builtin_expect(!keep_all, 0)) {
          const int nv = page_ok ? nvalid - 32 * ch : 0;
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = c < nv ? x[c] : -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) t[(c >> 1) & 3] = max3f(t[(c >> 1) & 3], x[c], x[c + 1]);
        mx = max3f(max3f(t[0], t[1], t[2]), t[3], t[3]);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = -INFINITY;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote_relaxed(lead_s_empty + 8u * sb);  // S was read (wait::ld)
      mx *= sl2;
      // the head's maximum over the whole tile: the other three threads of the head hold the rest
      // (double-buffered by tile parity: a buffer is rewritten only after the next exchange)
      tail->xmax[sb][lr][ch] = mx;
      // the four threads of a head are in warps w, w + 4, w ^ 2, (w ^ 2) + 4: warps of one parity
      named_barrier_sync(1 + (warp & 1), kSoftThreads / 2);
      {
        const float2 a = *reinterpret_cast<const float2*>(&tail->xmax[sb][lr][0]);
        const float2 b = *reinterpret_cast<const float2*>(&tail->xmax[sb][lr ^ 64][0]);
        mx = max3f(max3f(a.x, a.y, b.x), b.y, b.y);
      }
      // ---- the reference maximum, lazily raised ----
      const float m_prev = m_ref;
      float m_new = m_prev;
      if (m_prev == -INFINITY) m_new = mx;
      else if (mx > m_prev + kLazy) m_new = mx;
      const bool rescale = m_prev != -INFINITY && m_new > m_prev;  // O holds tiles so far
      const float mb = m_new == -INFINITY ? 0.f : m_new;
      if (rescale) l_own *= fast_exp2(m_prev - mb);
      m_ref = m_new;
      // P(i) goes into buffer i % 2, last read by P V(i-2)
      if (i >= 2) wwait(&tail->p_empty[sb], (uint32_t)(((i - 2) >> 1) & 1));
      // this thread's 32 weights of head hl: half of one 128-byte row of P's token chunk `half`, in
      // the 128-byte swizzled K-major layout the MMA reads (16-byte unit x of row r at x ^ (r % 8))
      uint8_t* prow = p_s + (size_t)sb * kPBytes + (size_t)half * (kHc * 128) + hl * 128;
      if (!dead) {
        uint32_t pk[16];
        float ps[8];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float z0, z1;
          fma2(z0, z1, x[c], x[c + 1], sl2, -mb);
          const float p0 = fast_exp2(z0), p1 = fast_exp2(z1);
          if (c < 8) ps[c] = p0, ps[c + 1] = p1;
          else add2(ps[c & 7], ps[(c & 7) + 1], p0, p1);
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        add2(ps[0], ps[1], ps[4], ps[5]);
        add2(ps[2], ps[3], ps[6], ps[7]);
        add2(ps[0], ps[1], ps[2], ps[3]);
        // O is normalised by the fp32 sum (the bf16-rounded weights differ from it by < 2^-9)
        l_own += ps[0] + ps[1];
#pragma unroll
        for (int xx = 0; xx < 4; ++xx)
          *reinterpret_cast<uint4*>(prow + (((4 * ch + xx) ^ (hl & 7)) << 4)) =
              make_uint4(pk[4 * xx], pk[4 * xx + 1], pk[4 * xx + 2], pk[4 * xx + 3]);
      }
      if (__builtin_expect(__any_sync(0xffffffffu, rescale) && !dead, 0)) {
        // O holds the segment's tiles < i: wait for P V(i-1), then rescale the rows that moved
        // (each thread of a head rescales its lane's columns 128 ch .. + 127), after P is written,
        // when the scores no longer take registers. P V(i) cannot start before this warp's P is
        // handed over, which comes after.
        wwait(&tail->p_empty[sb ^ 1], (uint32_t)(((i - 1) >> 1) & 1));
        const float alpha = rescale ? fast_exp2(m_prev - m_new) : 1.f;
        tc_fence_after();
        for (int c = 0; c < 128; c += 32) {
          float o[32];
          tmem_ld32(tl + kOCol + 128 * ch + c, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(tl + kOCol + 128 * ch + c, o);
        }
      }
      tc_fence_before();         // the O rescale before the MMA that reads it
      fence_proxy_async_smem();  // the generic-proxy P stores before the MMA's reads
      __syncwarp();
      if (lane == 0) arrive_remote(lead_p_full + 8u * sb);

      if (__builtin_expect(!seg_end, 1)) continue;
      // ---- end of a segment: O is complete once P V(i) is ----
      wwait(&tail->p_empty[sb], (uint32_t)((i >> 1) & 1));
      tc_fence_after();
      tail->xl[ch][lr] = l_own;
      named_barrier_sync(3, kSoftThreads);
      const float M = m_ref;  // the reference O and all four sums are relative to
      const float l_run = (tail->xl[0][lr] + tail->xl[1][lr]) + (tail->xl[0][lr ^ 64] + tail->xl[1][lr ^ 64]);
      const size_t orow = (size_t)urow[u] * kHeads + (size_t)rank * kHc + hl;
      const bool whole = g_begin <= pre[u] && g + 1 == pre[u + 1];
      float* rec = nullptr;
      if (!whole) {
        const int slot = (g_begin >= pre[u]) ? 0 : 1;
        rec = p.seg + (((size_t)pair * 2 + slot) * 2 + rank) * kRec;
      }
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      // TMEM lane lr, column block j = ch: value columns [256 j + 128 half, + 128) of head hl
      {
        const int j = ch;
        for (int c = 0; c < 128; c += 32) {
          float o[32];
          if (!dead) tmem_ld32(tl + kOCol + j * 128 + c, o);
          else
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = 0.f;
          const int col = 256 * j + 128 * half + c;
          float* dst = whole ? p.o_part + orow * kDV + col : rec + hl * kDV + col;
          const float f = whole ? inv : 1.f;
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + k) =
                make_float4(o[k] * f, o[k + 1] * f, o[k + 2] * f, o[k + 3] * f);
        }
      }
      tc_fence_before();
      if (whole) {
        if (half == 0 && ch == 0) p.lse[orow] = l_run > 0.f ? (M + log2f(l_run)) * kLn2 : -INFINITY;
      } else {
        if (half == 0 && ch == 0) {
          rec[kHc * kDV + hl] = M;
          rec[kHc * kDV + kHc + hl] = l_run;
          rec[kHc * kDV + 2 * kHc + hl] = l_run;
        }
        __threadfence();
        named_barrier_sync(3, kSoftThreads);
        const int c_lo = cta_of(pre[u], W, Geff), c_hi = cta_of((long long)pre[u + 1] - 1, W, Geff);
        if (lr == 0 && ch == 0) {
          const int ticket = atomicAdd(&p.tickets[u * 2 + rank], 1);
          tail->flag = ticket == c_hi - c_lo;
        }
        named_barrier_sync(3, kSoftThreads);
        if (tail->flag) {  // merge every cluster's segment of this unit, for this CTA's heads
          __threadfence();
          // segment c's record: the unit's first cluster used slot 1 unless its range started at
          // the unit's first tile; every later cluster's range starts inside the unit (slot 0)
          const int sl_lo = (range_begin(c_lo, W, Geff) >= pre[u]) ? 0 : 1;
          auto rec_of = [&](int c) {
            return p.seg + (((size_t)c * 2 + (c == c_lo ? sl_lo : 0)) * 2 + rank) * kRec;
          };
          float Mm = -INFINITY;
          for (int c = c_lo; c <= c_hi; ++c) Mm = fmaxf(Mm, __ldcg(rec_of(c) + kHc * kDV + hl));
          const float Mmu = Mm == -INFINITY ? 0.f : Mm;
          float Lm = 0.f, LBm = 0.f;
          for (int c = c_lo; c <= c_hi; ++c) {
            const float* rc = rec_of(c);
            const float w_ = fast_exp2(__ldcg(rc + kHc * kDV + hl) - Mmu);
            Lm += __ldcg(rc + kHc * kDV + kHc + hl) * w_;
            LBm += __ldcg(rc + kHc * kDV + 2 * kHc + hl) * w_;
          }
          const float invm = LBm > 0.f ? 1.f / LBm : 0.f;
          // this thread merges its quarter of the head's 512 columns, 16 columns at a time
          {
            const int j = ch;
            for (int c16 = 0; c16 < 128; c16 += 16) {
              const int col = 256 * j + 128 * half + c16;
              float4 acc[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
              for (int c = c_lo; c <= c_hi; ++c) {
                const float* rc = rec_of(c);
                const float w_ = fast_exp2(__ldcg(rc + kHc * kDV + hl) - Mmu);
                const float4* src = reinterpret_cast<const float4*>(rc + hl * kDV + col);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float4 v = __ldcg(src + k);
                  acc[k].x += v.x * w_;
                  acc[k].y += v.y * w_;
                  acc[k].z += v.z * w_;
                  acc[k].w += v.w * w_;
                }
              }
              float4* dst = reinterpret_cast<float4*>(p.o_part + orow * kDV + col);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_float4(acc[k].x * invm, acc[k].y * invm, acc[k].z * invm,
                                     acc[k].w * invm);
            }
          }
          if (half == 0 && ch == 0) p.lse[orow] = Lm > 0.f ? (Mm + log2f(Lm)) * kLn2 : -INFINITY;
          named_barrier_sync(3, kSoftThreads);
          if (lr == 0 && ch == 0) p.tickets[u * 2 + rank] = 0;
        }
      }
    }
  }

  // ---- teardown: every thread of both CTAs gets here (all waits above are bounded) ----
  if (warp == kMmaWarp && lane == 0) {
    // every pair-wide MMA has completed before TMEM is released (bounded: on a timeout the kernel
    // has already reported an error)
    if (!mbar_wait_pair(&tail->mma_done, 0)) raise_dev_error(p.err, HELIX_DEVERR_WAIT_TIMEOUT);
  }
  if (*(volatile int*)&tail->abort_) {
    // after a wait ran out, loads issued before it may still be landing: give them time
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 200000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote arrival, load completion or MMA targets this CTA after this
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

size_t mla_partial_smem_bytes(int units) {
  return kSmemFixed + (size_t)(3 * units + 1) * sizeof(int);  // pre, urow, ulen
}
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
