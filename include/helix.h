/*
 * helix.h -- C ABI of libhelix.so: KV-parallel (sequence-sharded) decode attention on one B200.
 *
 * The method ("Helix Parallelism: Rethinking Sharding Strategies for Interactive Multi-Million-Token
 * LLM Decoding"; paper summary page, fdeinterviews.com, paragraph on KV parallelism): the KV history
 * of every request is split along the sequence into KVP shards. For one new query token each shard
 * attends over its own slice and returns a partial output plus the log-sum-exp (LSE) of its logits;
 * an LSE-rescaling combine then yields exactly the full-context result. On one GPU the shards are
 * partitions of one paged pool in HBM, and the combine reads the partials from HBM where the
 * multi-GPU system would run an all-to-all.
 *
 * Three calls make one decode-attention layer step:
 *   helix_kv_append     place the new token's K/V round-robin across shards (16-token blocks)
 *   helix_attn_partial  per-shard partial attention -> O_partial[shard][B][Hq][dv], lse[shard][B][Hq]
 *   helix_attn_combine  O = sum_s exp(lse_s - LSE) * O_s, LSE = log sum_s exp(lse_s)
 *
 * Conventions (all calls):
 *  - Every pointer argument that names tensor data is DEVICE memory owned by the caller; the
 *    library never allocates, frees or retains it beyond the call. Scratch space for the partial
 *    call is a caller-provided workspace (size from helix_attn_workspace_size).
 *  - Every call is asynchronous on `stream` (NULL = the legacy default stream). Host-side argument
 *    validation happens before any launch: on error the call returns a status and launches nothing.
 *  - Conditions only the device can see (a page id outside the pool, a history longer than the
 *    page table) set bits in the optional `*err_word` of the cache (HELIX_DEVERR_*), skip the
 *    affected work and never trap. The caller reads err_word after synchronising.
 *  - A failed launch returns HELIX_ERR_CUDA. No C++ exception crosses this interface.
 *  - Tensors are dense, row-major, with the shapes given below; every base pointer must be 16-byte
 *    aligned.
 *  - Calls that share a workspace or a cache must be ordered on one stream (or by events).
 */
#ifndef HELIX_H_
#define HELIX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared opaquely so this header needs no CUDA headers. */
typedef struct CUstream_st* helix_stream_t;
typedef struct CUevent_st* helix_event_t; /* a cudaEvent_t */

typedef enum {
  HELIX_OK = 0,
  HELIX_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misaligned pointer, workspace too small */
  HELIX_ERR_UNSUPPORTED = 2, /* a shape/dtype combination no kernel is built for */
  HELIX_ERR_CAPACITY = 3,    /* the call cannot fit its work in the sizes given */
  HELIX_ERR_CUDA = 4,        /* a CUDA runtime error (launch failure, no device, ...) */
  HELIX_ERR_TIMEOUT = 5      /* a host-side wait with a limit ran out (helix_stream_wait) */
} helix_status;

/* Bits written (OR-ed) into *err_word by the kernels. */
#define HELIX_DEVERR_PAGE_ID 0x1u      /* page_table entry < 0 or >= num_pages: page skipped */
#define HELIX_DEVERR_CAPACITY 0x2u     /* a local index past max_pages_per_shard pages: skipped */
#define HELIX_DEVERR_SHARD 0x4u        /* contiguous layout placed a token past the last shard */
#define HELIX_DEVERR_WAIT_TIMEOUT 0x8u /* an on-chip pipeline wait ran out of its limit */

typedef enum { HELIX_KV_BF16 = 0, HELIX_KV_NVFP4 = 1 } helix_kv_dtype;
typedef enum { HELIX_ATTN_GQA = 0, HELIX_ATTN_MLA = 1 } helix_attn_kind;
typedef enum { HELIX_LAYOUT_RR = 0, HELIX_LAYOUT_CONTIG = 1 } helix_layout;

/*
 * The paged, sequence-sharded KV cache of one attention layer.
 *
 * Placement of history token t (0-based global position) of request b:
 *   HELIX_LAYOUT_RR (paper summary, paragraph on the Helix layouts; NVIDIA technical blog, Korean
 *   edition, KV-cache section, round-robin example): block j = t / rr_block goes to shard
 *   s = j % kvp, at local index l = (j / kvp) * rr_block + t % rr_block.
 *   HELIX_LAYOUT_CONTIG: s = t / contig_chunk, l = t % contig_chunk.
 * Local index l is stored in page page_table[s][b][l / page_tokens] at slot l % page_tokens.
 *
 * Pool layouts (P = num_pages, H = num_kv_heads, T = page_tokens, d = head_dim):
 *   GQA, BF16 : k_pool, v_pool  bf16  [P][H][T][d]
 *   GQA, NVFP4: k_pool  uint8 [P][H][T][d/2]  E2M1 codes of K, element 2i in the low nibble
 *               k_scale uint8 [P][H][T][d/16] E4M3 scale of elements 16j..16j+15 of a K row
 *               v_pool  uint8 [P][H][T/2][d]  E2M1 codes of V, token-pair interleaved: the byte
 *                       for (pair i, column c) holds V[token 2i][c] in the low nibble and
 *                       V[token 2i+1][c] in the high nibble (the P.V contraction runs over tokens,
 *                       so its operands pair tokens); within pair row i it sits at byte
 *                       16 * ((c / 16) XOR (2 * (i mod 4))) + c mod 16 (a bank-conflict swizzle)
 *               v_scale uint8 [P][H][d/16][T] E4M3 scale of elements 16j..16j+15 of V row t, at [j][t]
 *               helix_kv_append takes K and V rows in the same natural row format and does the
 *               V re-layout.
 *   MLA, BF16 : k_pool          bf16  [P][T][d] with d = 576 (H = 1); V is columns [0, v_dim) of
 *               the same rows (v_pool must be NULL): keys and values share one latent row.
 *
 * State updated by helix_kv_append: seq_lens[b] (history length of request b) and
 * shard_lens[s][b] (tokens shard s holds for request b). helix_attn_partial reads shard_lens.
 */
typedef struct helix_kv_cache {
  int32_t kind;                /* helix_attn_kind */
  int32_t kv_dtype;            /* helix_kv_dtype */
  int32_t layout;              /* helix_layout */
  int32_t kvp;                 /* number of KV-parallel shards, >= 1 */
  int32_t batch;               /* requests B */
  int32_t num_kv_heads;        /* Hkv (GQA); 1 for MLA */
  int32_t head_dim;            /* d: 64 or 128 (GQA), 576 (MLA) */
  int32_t v_dim;               /* dv: = head_dim (GQA), 512 (MLA) */
  int32_t page_tokens;         /* tokens per page; 64 */
  int32_t rr_block;            /* round-robin block; 16 */
  int32_t contig_chunk;        /* tokens per shard, HELIX_LAYOUT_CONTIG only */
  int32_t num_pages;           /* pages in the pool */
  int32_t max_pages_per_shard; /* third extent of page_table */
  int32_t reserved_;
  void* k_pool;
  void* v_pool;
  void* k_scale;
  void* v_scale;
  const int32_t* page_table; /* int32 [kvp][batch][max_pages_per_shard] */
  int32_t* shard_lens;       /* int32 [kvp][batch] */
  int32_t* seq_lens;         /* int32 [batch] */
  uint32_t* err_word;        /* optional (may be NULL): HELIX_DEVERR_* bits are OR-ed in */
} helix_kv_cache;

/*
 * Append up to n_new tokens to every request. Row j of request b's slice gets global position
 * seq_lens[b] + j and is placed by the cache's layout rule. Afterwards seq_lens[b] grows by the
 * number of rows appended and shard_lens[s][b] by the number of them placed on shard s.
 *   GQA BF16 : k_new, v_new bf16 [B][n_new][H][d]; k_new_scale = v_new_scale = NULL
 *   GQA NVFP4: k_new, v_new uint8 [B][n_new][H][d/2]; k_new_scale, v_new_scale uint8 [B][n_new][H][d/16]
 *   MLA      : k_new bf16 [B][n_new][576]; v_new = NULL
 *   n_valid  : optional device int32 [B]; when given, request b appends only its first
 *              min(max(n_valid[b], 0), n_new) rows (ragged prefill). NULL = n_new rows each.
 * The copy is bit-exact. n_new = 0 is a no-op. Device errors: HELIX_DEVERR_PAGE_ID, _CAPACITY,
 * _SHARD (the row is not stored; the lengths still advance).
 */
helix_status helix_kv_append(const helix_kv_cache* cache, const void* k_new, const void* v_new,
                             const void* k_new_scale, const void* v_new_scale, int32_t n_new,
                             const int32_t* n_valid, helix_stream_t stream);

/*
 * helix_kv_append for an NVFP4 GQA cache (head_dim 128) from bf16 rows, encoding on the device:
 *   k_new, v_new bf16 [B][n_new][H][128] (16-byte aligned); n_valid as in helix_kv_append.
 * Each 16-element block of a row gets scale = the E4M3 value nearest to fp32(absmax / 6) (ties to
 * even, clamped to 448) and codes = the E2M1 values nearest to fp32(x / scale) (x itself when the
 * scale is 0; ties to even, saturating at 6; a value rounding to zero is stored as +0), every
 * division in IEEE fp32. The pages say only "FP4"; the block size, scale type and absmax / 6 rule
 * are those of the NVFP4 format. Placement, lengths and device errors as helix_kv_append.
 * Returns HELIX_ERR_UNSUPPORTED for other cache kinds.
 */
helix_status helix_kv_append_quantize(const helix_kv_cache* cache, const void* k_new,
                                      const void* v_new, int32_t n_new, const int32_t* n_valid,
                                      helix_stream_t stream);

/*
 * Bytes of workspace helix_attn_partial needs for this cache shape on the current device.
 * The workspace must be zero-filled once before its first use; the kernel returns it to that
 * state, so later calls need no clearing (unless a previous call was aborted by a device error).
 */
helix_status helix_attn_workspace_size(const helix_kv_cache* cache, int32_t num_q_heads,
                                       size_t* bytes);

/*
 * Per-shard partial attention for one new query token per request (paper summary, paragraph on
 * KV parallelism: each shard attends over its slice and returns a partial output plus an LSE).
 *   q          bf16  [B][num_q_heads][head_dim]
 *   o_partial  fp32  [kvp][B][num_q_heads][v_dim]  O_s = softmax-weighted V over shard s's tokens,
 *                                                  normalised over those tokens
 *   lse        fp32  [kvp][B][num_q_heads]          natural-log LSE of shard s's scaled logits
 * Logit of head h against token t: softmax_scale * <q[b][h], K[t][h / (num_q_heads / H)]>.
 * A shard with no tokens gives O_s = 0 and lse = -inf.
 * GQA: num_q_heads % H == 0 and num_q_heads / H <= 16. MLA: num_q_heads == 128.
 * Work is enqueued on `stream` as one kernel launch, except for MLA batches with more (request,
 * shard) units than one launch keeps in shared memory (about 570 on a B200): those run as
 * consecutive launches over request ranges, sharing the workspace, with the same results.
 * HELIX_ERR_CAPACITY only if one request's units do not fit.
 */
helix_status helix_attn_partial(const helix_kv_cache* cache, const void* q, int32_t num_q_heads,
                                float softmax_scale, float* o_partial, float* lse, void* workspace,
                                size_t workspace_bytes, helix_stream_t stream);

/*
 * LSE-rescaling combine (paper review, jaehun.me, "Prompt 1.3.2 -- The Secret Weapon", boxed
 * equation, read for partials normalised per shard): for every (b, h)
 *   M = max_s lse_s,  LSE = M + ln sum_s exp(lse_s - M),  O = sum_s exp(lse_s - LSE) * O_s.
 * Shards with lse = -inf carry no weight; if all are -inf, O = 0 and LSE = -inf.
 *   o_partial fp32 [kvp][batch][num_q_heads][v_dim], lse fp32 [kvp][batch][num_q_heads]
 *   o_out     [batch][num_q_heads][v_dim], bf16 (o_dtype 0) or fp32 (o_dtype 1)
 *   lse_out   fp32 [batch][num_q_heads], may be NULL
 * v_dim must be a multiple of 4.
 */
helix_status helix_attn_combine(int32_t kvp, int32_t batch, int32_t num_q_heads, int32_t v_dim,
                                const float* o_partial, const float* lse, void* o_out,
                                int32_t o_dtype, float* lse_out, helix_stream_t stream);

/*
 * The same combine over partials held in separate buffers, one per source shard, for the heads
 * [head_begin, head_end) of every request. This is the owner's side of the exchange between GPUs
 * (paper summary: after attention, an all-to-all takes the partial outputs and LSEs of every KV
 * shard to the rank that owns a head group): on a multi-GPU node o_parts[s] / lses[s] are the
 * source ranks' own buffers mapped into this process (CUDA IPC), read with plain loads over NVLink,
 * so the exchange and the merge are one kernel.
 *   o_parts[s]  fp32 [batch][num_q_heads][v_dim], lses[s] fp32 [batch][num_q_heads], s < nsrc
 *               (host arrays of device-accessible pointers; 16-byte / 4-byte aligned)
 *   o_out       [batch][head_end - head_begin][v_dim], bf16 (o_dtype 0) or fp32 (o_dtype 1)
 *   lse_out     fp32 [batch][head_end - head_begin], may be NULL
 * 1 <= nsrc <= HELIX_MAX_SOURCES; v_dim a multiple of 4. The arithmetic is helix_attn_combine's, in
 * the same order: the results are bit-identical to it for the same partials.
 */
#define HELIX_MAX_SOURCES 16
helix_status helix_attn_combine_sources(int32_t nsrc, const float* const* o_parts,
                                        const float* const* lses, int32_t batch,
                                        int32_t num_q_heads, int32_t v_dim, int32_t head_begin,
                                        int32_t head_end, void* o_out, int32_t o_dtype,
                                        float* lse_out, helix_stream_t stream);

/*
 * helix_attn_partial followed by helix_attn_combine, in ONE launch for GQA caches: the CTA that
 * finishes the last of the kvp shards of a (request, KV head) group merges that group's rows into
 * o_out / lse_out in the same kernel (the same arithmetic as helix_attn_combine, bit for bit).
 * o_partial / lse still receive the per-shard results. For MLA caches the merge of a request
 * (128 x 512 per shard) is too large for one CTA and this call issues the two launches.
 *   arguments as helix_attn_partial + helix_attn_combine (o_dtype 0 bf16, 1 fp32; lse_out may be
 *   NULL); the workspace is the one helix_attn_workspace_size reports.
 * This is the step the paper summary describes for short contexts too (below about 4K tokens Helix
 * degenerates to data-parallel attention): with kvp = 1 the merge is the identity and the step is
 * one launch.
 */
helix_status helix_attn_partial_combine(const helix_kv_cache* cache, const void* q,
                                        int32_t num_q_heads, float softmax_scale,
                                        float* o_partial, float* lse, void* o_out,
                                        int32_t o_dtype, float* lse_out, void* workspace,
                                        size_t workspace_bytes, helix_stream_t stream);

/*
 * helix_attn_partial restricted to the requests [b_begin, b_end) (0 <= b_begin <= b_end <= batch).
 * q, o_partial and lse keep their full shapes and indexing; rows of other requests are neither read
 * nor written. Same workspace as helix_attn_partial: calls sharing a workspace must be ordered on
 * the GPU (one stream, or events). b_begin == b_end launches nothing.
 */
helix_status helix_attn_partial_range(const helix_kv_cache* cache, const void* q,
                                      int32_t num_q_heads, float softmax_scale, int32_t b_begin,
                                      int32_t b_end, float* o_partial, float* lse, void* workspace,
                                      size_t workspace_bytes, helix_stream_t stream);

/* helix_attn_combine restricted to the requests [b_begin, b_end); full-shape arrays as above. */
helix_status helix_attn_combine_range(int32_t kvp, int32_t batch, int32_t num_q_heads,
                                      int32_t v_dim, int32_t b_begin, int32_t b_end,
                                      const float* o_partial, const float* lse, void* o_out,
                                      int32_t o_dtype, float* lse_out, helix_stream_t stream);

/*
 * One-GPU analogue of HOP-B, the batch-wise overlap of one request's exchange with the next
 * request's attention (ifai.io news, "Decoupling attention and FFN"; NVIDIA blog, Korean edition,
 * Figure 3). The batch is cut into n_groups contiguous request groups (ceil(B / n_groups) requests
 * each; n_groups is clamped to B). On stream_a the partial attention of group g runs after that of
 * group g-1 (they share the workspace); on stream_b the combine of group g waits for it (event
 * events[g]) and then overlaps the partial of group g+1. Finally stream_a waits for stream_b
 * (events[n_groups]), so the results are ready when stream_a's work is.
 *   events : n_groups + 1 CUDA events created by the caller (timing disabled is best)
 *   other arguments as helix_attn_partial + helix_attn_combine (o_dtype 0 bf16, 1 fp32;
 *   lse_out may be NULL). stream_a and stream_b must differ.
 * Results equal helix_attn_partial_range over each group followed by the combine: per request, the
 * same numbers up to the rounding of how the kernel splits a group's units across CTAs.
 * Every argument is validated before the first launch.
 */
helix_status helix_attn_overlapped(const helix_kv_cache* cache, const void* q, int32_t num_q_heads,
                                   float softmax_scale, int32_t n_groups, float* o_partial,
                                   float* lse, void* o_out, int32_t o_dtype, float* lse_out,
                                   void* workspace, size_t workspace_bytes,
                                   helix_stream_t stream_a, helix_stream_t stream_b,
                                   const helix_event_t* events);

/*
 * The HOP-B analogue for a whole decode step: as helix_attn_overlapped, and the append of each
 * request group's new tokens also runs on stream_b, overlapping the previous group's partial
 * attention (the pages' batch-wise overlap, extended to the append).
 *   k_new ... n_new  as helix_kv_append (all requests' rows);
 *   group_n_valid    device int32 [min(n_groups, B)][B]: row g gives every request's number of
 *                    new rows for group g's append (n_new for requests of group g, 0 otherwise;
 *                    groups are contiguous, ceil(B / n_groups) requests each);
 *   events           2 * min(n_groups, B) + 1 caller-created CUDA events.
 * Order: B: append(0); then per group g: A waits for append(g), runs partial(g); B runs
 * append(g+1), waits for partial(g), runs combine(g); finally A waits for B. Requests whose row has
 * 0 new tokens are not touched by that append (their lengths are not even rewritten).
 */
helix_status helix_decode_overlapped(const helix_kv_cache* cache, const void* q,
                                    int32_t num_q_heads, float softmax_scale, int32_t n_groups,
                                    const void* k_new, const void* v_new, const void* k_new_scale,
                                    const void* v_new_scale, int32_t n_new,
                                    const int32_t* group_n_valid, float* o_partial, float* lse,
                                    void* o_out, int32_t o_dtype, float* lse_out, void* workspace,
                                    size_t workspace_bytes, helix_stream_t stream_a,
                                    helix_stream_t stream_b, const helix_event_t* events);

/*
 * helix_attn_partial for callers that cannot allocate device memory. The paper has no counterpart;
 * this is a deployment convenience of this library.
 *
 * Same arguments and results as helix_attn_partial, minus the workspace: the kernel's scratch lives
 * in a fixed device array of HELIX_NOALLOC_SCRATCH_BYTES inside the library (one per GPU, held
 * until the process exits). Meant for code that has no way to obtain a scratch buffer -- a plugin
 * whose host owns all device memory, a fixed pre-reserved memory budget, or a loop that must never
 * call cudaMalloc. The call allocates nothing.
 *   - Returns HELIX_ERR_CAPACITY, launching nothing, when this cache shape needs more scratch than
 *     HELIX_NOALLOC_SCRATCH_BYTES (see helix_attn_workspace_size).
 *   - Every argument is checked before anything is enqueued: a rejected call launches nothing and
 *     does not touch the shared array.
 *   - The first call on each device looks up the array's device address (once, with that device
 *     current); make that first call before any stream capture. The address is kept for the life
 *     of the process: after cudaDeviceReset on a device, do not call this entry point there again.
 *   - Each call zeroes the scratch it uses (an async memset on `stream`) before the kernel runs.
 *   - All calls on one device share the array: calls that may run concurrently on the GPU race and
 *     must be ordered by the caller (one stream, or events).
 */
/* 48 MiB: an MLA cache needs about 37 MiB of split-unit records on a 148-SM B200 (2 per cluster of
 * 2 CTAs, 64 heads x 515 floats each per CTA), a GQA cache about 2.5 MB. */
#define HELIX_NOALLOC_SCRATCH_BYTES (48u << 20)
helix_status helix_attn_partial_noalloc(const helix_kv_cache* cache, const void* q,
                                        int32_t num_q_heads, float softmax_scale,
                                        float* o_partial, float* lse, helix_stream_t stream);

/*
 * Wait, with a wall-clock limit, for the work enqueued on `stream` so far. The library has no
 * counterpart in the pages; this is the host side of its failure handling: where
 * cudaStreamSynchronize would block for as long as the GPU takes, this call records `event` on
 * `stream` and polls it (cudaEventQuery) until the work is done or `limit_us` microseconds have
 * passed.
 *   event    a CUDA event created by the caller (timing disabled is best); re-recorded here.
 *   limit_us the limit in microseconds (0 polls once).
 * Returns HELIX_OK when all of the stream's earlier work has finished, HELIX_ERR_TIMEOUT when the
 * limit passed first (the work is still enqueued and may finish later: the caller decides whether
 * to wait again or give up), HELIX_ERR_CUDA when recording or querying the event fails (including
 * an error raised by the stream's earlier work), HELIX_ERR_INVALID_ARG for a NULL event.
 */
helix_status helix_stream_wait(helix_stream_t stream, helix_event_t event, uint64_t limit_us);

/* Static, human-readable name of a status code. */
const char* helix_status_string(helix_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t helix_version(void);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* HELIX_H_ */
