// abi.cu -- the extern "C" entry points of libhelix.so: argument validation, TMA descriptor
// encoding and dispatch to the kernels. Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "bounded_wait.h"
#include "helix.h"
#include "internal.h"

namespace helix {
namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over a pool viewed as [rows][row_elems] with 64 x box_rows boxes, 128-byte swizzle.
bool encode_rows_map(CUtensorMap* map, void* base, CUtensorMapDataType dt, int elem_bytes,
                     uint64_t row_elems, uint64_t rows, uint32_t box_elems, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {row_elems, rows};
  const cuuint64_t strides[1] = {row_elems * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {box_elems, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The MLA latent pool (bf16 rows of 576) seen as a 3-D tensor [9 chunks][rows][64 columns]: the
// chunk dimension has a stride of 128 bytes (one chunk of a row), so one box of 64 columns x 64 rows
// x 2 chunks lands in shared memory as two consecutive 64-row chunk tiles in the 128-byte swizzled
// layout the tensor cores read.
bool encode_latent_chunks_map(CUtensorMap* map, void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {64, rows, 9};
  const cuuint64_t strides[2] = {576 * 2, 64 * 2};
  const cuuint32_t box[3] = {64, 64, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return 0;
}

int device_max_smem(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(out, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return -1;
  return 0;
}

// Shape checks common to every call that takes a cache.
helix_status check_cache(const helix_kv_cache* c) {
  if (c == nullptr) return HELIX_ERR_INVALID_ARG;
  if (c->kvp < 1 || c->batch < 1 || c->num_kv_heads < 1 || c->head_dim < 1 || c->v_dim < 1 ||
      c->page_tokens < 1 || c->num_pages < 1 || c->max_pages_per_shard < 1)
    return HELIX_ERR_INVALID_ARG;
  if (c->layout == HELIX_LAYOUT_RR) {
    if (c->rr_block < 1) return HELIX_ERR_INVALID_ARG;
  } else if (c->layout == HELIX_LAYOUT_CONTIG) {
    if (c->contig_chunk < 1) return HELIX_ERR_INVALID_ARG;
  } else {
    return HELIX_ERR_INVALID_ARG;
  }
  if (c->page_table == nullptr || c->shard_lens == nullptr || c->seq_lens == nullptr)
    return HELIX_ERR_INVALID_ARG;
  if (!aligned4(c->page_table) || !aligned4(c->shard_lens) || !aligned4(c->seq_lens) ||
      !aligned4(c->err_word))
    return HELIX_ERR_INVALID_ARG;
  if (c->k_pool == nullptr || !aligned16(c->k_pool)) return HELIX_ERR_INVALID_ARG;
  if (c->kind == HELIX_ATTN_GQA) {
    if (c->v_pool == nullptr || !aligned16(c->v_pool)) return HELIX_ERR_INVALID_ARG;
    if (c->v_dim != c->head_dim) return HELIX_ERR_INVALID_ARG;
    if (c->kv_dtype == HELIX_KV_NVFP4) {
      if (c->head_dim != 128) return HELIX_ERR_UNSUPPORTED;  // the V-code swizzle spans 8 chunks
      if (c->k_scale == nullptr || c->v_scale == nullptr || !aligned16(c->k_scale) ||
          !aligned16(c->v_scale))
        return HELIX_ERR_INVALID_ARG;
    } else if (c->kv_dtype != HELIX_KV_BF16) {
      return HELIX_ERR_INVALID_ARG;
    }
  } else if (c->kind == HELIX_ATTN_MLA) {
    if (c->num_kv_heads != 1 || c->v_pool != nullptr || c->kv_dtype != HELIX_KV_BF16 ||
        c->v_dim > c->head_dim)
      return HELIX_ERR_INVALID_ARG;
  } else {
    return HELIX_ERR_INVALID_ARG;
  }
  // pool rows, local indices and prefix sums are 32-bit on the device
  const int64_t rows = (int64_t)c->num_pages * c->num_kv_heads * c->page_tokens;
  const int64_t units = (int64_t)c->batch * c->num_kv_heads * c->kvp;
  if (rows > INT32_MAX || units * c->max_pages_per_shard > INT32_MAX ||
      (int64_t)c->max_pages_per_shard * c->page_tokens > INT32_MAX)
    return HELIX_ERR_CAPACITY;
  return HELIX_OK;
}

// Workspace layout: [unit tickets][group tickets (GQA fused combine)][segment records]
struct PartialPlan {
  int grid;
  int units;
  int max_units;  // units one launch can take (a multiple of the units per request)
  size_t ticket_bytes;
  size_t gticket_bytes;
  size_t seg_bytes;
  size_t total() const { return ticket_bytes + gticket_bytes + seg_bytes; }
};

helix_status plan_partial(const helix_kv_cache* c, int num_q_heads, PartialPlan* plan) {
  helix_status st = check_cache(c);
  if (st != HELIX_OK) return st;
  if (num_q_heads < 1 || num_q_heads % c->num_kv_heads != 0) return HELIX_ERR_INVALID_ARG;
  if (c->page_tokens != 64) return HELIX_ERR_UNSUPPORTED;
  if (c->kind == HELIX_ATTN_MLA) {
    // one kernel shape: 128 heads against a 576-wide latent whose first 512 columns are V
    if (num_q_heads != 128 || c->head_dim != 576 || c->v_dim != 512) return HELIX_ERR_UNSUPPORTED;
    int sms = 0, max_smem = 0;
    if (device_sm_count(&sms) != 0 || device_max_smem(&max_smem) != 0) return HELIX_ERR_CUDA;
    plan->units = c->batch * c->kvp;
    // a launch keeps three ints per unit (tile prefix sum, shard row, length) in shared memory:
    // a batch whose units do not fit is run as consecutive launches over request ranges
    if (mla_partial_smem_bytes(0) > (size_t)max_smem) return HELIX_ERR_CAPACITY;
    const size_t room = ((size_t)max_smem - mla_partial_smem_bytes(0)) / (3 * sizeof(int));
    const int fit = room < (size_t)plan->units ? (int)room : plan->units;
    plan->max_units = (fit / c->kvp) * c->kvp;
    if (plan->max_units < c->kvp) return HELIX_ERR_CAPACITY;
    plan->grid = (sms / 2) * 2;  // clusters of two CTAs
    if (plan->grid < 2) return HELIX_ERR_UNSUPPORTED;
    plan->ticket_bytes = (((size_t)plan->units * 2 * sizeof(int32_t)) + 255) & ~size_t(255);
    plan->gticket_bytes = 0;
    plan->seg_bytes = (size_t)(plan->grid / 2) * 2 * 2 * mla_segment_record_floats() * sizeof(float);
    return HELIX_OK;
  }
  if (c->kind != HELIX_ATTN_GQA) return HELIX_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return HELIX_ERR_UNSUPPORTED;
  if (num_q_heads / c->num_kv_heads > 16) return HELIX_ERR_UNSUPPORTED;
  const int nvfp4 = c->kv_dtype == HELIX_KV_NVFP4;
  if (nvfp4 && c->head_dim != 128) return HELIX_ERR_UNSUPPORTED;
  int sms = 0, max_smem = 0;
  if (device_sm_count(&sms) != 0 || device_max_smem(&max_smem) != 0) return HELIX_ERR_CUDA;
  plan->units = c->batch * c->num_kv_heads * c->kvp;
  const size_t smem = nvfp4 ? gqa_nvfp4_smem_bytes(plan->units)
                            : gqa_partial_smem_bytes(c->head_dim, plan->units);
  if (smem > (size_t)max_smem) return HELIX_ERR_CAPACITY;
  plan->max_units = plan->units;
  plan->grid = sms;
  plan->ticket_bytes = (((size_t)plan->units * sizeof(int32_t)) + 255) & ~size_t(255);
  plan->gticket_bytes =
      (((size_t)c->batch * c->num_kv_heads * sizeof(int32_t)) + 255) & ~size_t(255);
  const size_t rec = nvfp4 ? gqa_nvfp4_segment_record_floats()
                           : gqa_segment_record_floats(c->head_dim);
  plan->seg_bytes = (size_t)plan->grid * 2 * rec * sizeof(float);
  return HELIX_OK;
}

}  // namespace
}  // namespace helix

using namespace helix;

extern "C" {

const char* helix_status_string(helix_status s) {
  switch (s) {
    case HELIX_OK: return "HELIX_OK";
    case HELIX_ERR_INVALID_ARG: return "HELIX_ERR_INVALID_ARG";
    case HELIX_ERR_UNSUPPORTED: return "HELIX_ERR_UNSUPPORTED";
    case HELIX_ERR_CAPACITY: return "HELIX_ERR_CAPACITY";
    case HELIX_ERR_CUDA: return "HELIX_ERR_CUDA";
    case HELIX_ERR_TIMEOUT: return "HELIX_ERR_TIMEOUT";
  }
  return "HELIX_ERR_UNKNOWN";
}

int32_t helix_version(void) { return kVersion; }

helix_status helix_kv_append(const helix_kv_cache* c, const void* k_new, const void* v_new,
                             const void* k_new_scale, const void* v_new_scale, int32_t n_new,
                             const int32_t* n_valid, helix_stream_t stream) {
  helix_status st = check_cache(c);
  if (st != HELIX_OK) return st;
  if (n_new < 0) return HELIX_ERR_INVALID_ARG;
  if (n_new == 0) return HELIX_OK;
  AppendParams p{};
  const int d = c->head_dim;
  if (c->kind == HELIX_ATTN_GQA && c->kv_dtype == HELIX_KV_BF16) {
    if (k_new == nullptr || v_new == nullptr || !aligned4(k_new) || !aligned4(v_new))
      return HELIX_ERR_INVALID_ARG;
    p.src[0] = (const uint8_t*)k_new; p.dst[0] = (uint8_t*)c->k_pool; p.row_bytes[0] = d * 2;
    p.src[1] = (const uint8_t*)v_new; p.dst[1] = (uint8_t*)c->v_pool; p.row_bytes[1] = d * 2;
  } else if (c->kind == HELIX_ATTN_GQA && c->kv_dtype == HELIX_KV_NVFP4) {
    if (k_new == nullptr || v_new == nullptr || k_new_scale == nullptr || v_new_scale == nullptr ||
        !aligned4(k_new) || !aligned4(v_new) || !aligned4(k_new_scale) || !aligned4(v_new_scale))
      return HELIX_ERR_INVALID_ARG;
    p.src[0] = (const uint8_t*)k_new; p.dst[0] = (uint8_t*)c->k_pool; p.row_bytes[0] = d / 2;
    p.src[1] = (const uint8_t*)v_new; p.dst[1] = (uint8_t*)c->v_pool; p.row_bytes[1] = d / 2;
    p.src[2] = (const uint8_t*)k_new_scale; p.dst[2] = (uint8_t*)c->k_scale; p.row_bytes[2] = d / 16;
    p.src[3] = (const uint8_t*)v_new_scale; p.dst[3] = (uint8_t*)c->v_scale; p.row_bytes[3] = d / 16;
    p.v_nvfp4 = 1;
    if (c->page_tokens % 2 != 0 || d % 8 != 0) return HELIX_ERR_INVALID_ARG;
  } else {  // MLA: one latent row per token, V aliases its first v_dim columns
    if (k_new == nullptr || v_new != nullptr || !aligned4(k_new)) return HELIX_ERR_INVALID_ARG;
    p.src[0] = (const uint8_t*)k_new; p.dst[0] = (uint8_t*)c->k_pool; p.row_bytes[0] = d * 2;
  }
  p.page_table = c->page_table;
  p.shard_lens = c->shard_lens;
  p.seq_lens = c->seq_lens;
  p.err = c->err_word;
  p.B = c->batch;
  p.Hkv = c->num_kv_heads;
  p.kvp = c->kvp;
  p.layout = c->layout;
  p.rr_block = c->rr_block;
  p.contig_chunk = c->contig_chunk;
  p.page_tokens = c->page_tokens;
  p.max_pages = c->max_pages_per_shard;
  p.num_pages = c->num_pages;
  p.n_new = n_new;
  if (!aligned4(n_valid)) return HELIX_ERR_INVALID_ARG;
  p.n_valid = n_valid;
  return append_launch(p, reinterpret_cast<cudaStream_t>(stream));
}

helix_status helix_kv_append_quantize(const helix_kv_cache* c, const void* k_new,
                                      const void* v_new, int32_t n_new, const int32_t* n_valid,
                                      helix_stream_t stream) {
  helix_status st = check_cache(c);
  if (st != HELIX_OK) return st;
  if (c->kind != HELIX_ATTN_GQA || c->kv_dtype != HELIX_KV_NVFP4) return HELIX_ERR_UNSUPPORTED;
  if (c->head_dim != 128 || c->page_tokens % 2 != 0) return HELIX_ERR_UNSUPPORTED;
  if (n_new < 0) return HELIX_ERR_INVALID_ARG;
  if (n_new == 0) return HELIX_OK;
  if (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned4(n_valid))
    return HELIX_ERR_INVALID_ARG;
  AppendParams p{};
  p.src[0] = (const uint8_t*)k_new; p.dst[0] = (uint8_t*)c->k_pool; p.row_bytes[0] = 256;
  p.src[1] = (const uint8_t*)v_new; p.dst[1] = (uint8_t*)c->v_pool; p.row_bytes[1] = 256;
  p.dst[2] = (uint8_t*)c->k_scale;
  p.dst[3] = (uint8_t*)c->v_scale;
  p.quantize = 1;
  p.v_nvfp4 = 1;
  p.page_table = c->page_table;
  p.shard_lens = c->shard_lens;
  p.seq_lens = c->seq_lens;
  p.err = c->err_word;
  p.B = c->batch;
  p.Hkv = c->num_kv_heads;
  p.kvp = c->kvp;
  p.layout = c->layout;
  p.rr_block = c->rr_block;
  p.contig_chunk = c->contig_chunk;
  p.page_tokens = c->page_tokens;
  p.max_pages = c->max_pages_per_shard;
  p.num_pages = c->num_pages;
  p.n_new = n_new;
  p.n_valid = n_valid;
  return append_launch(p, reinterpret_cast<cudaStream_t>(stream));
}

helix_status helix_attn_workspace_size(const helix_kv_cache* c, int32_t num_q_heads,
                                       size_t* bytes) {
  if (bytes == nullptr) return HELIX_ERR_INVALID_ARG;
  PartialPlan plan;
  helix_status st = plan_partial(c, num_q_heads, &plan);
  if (st != HELIX_OK) return st;
  *bytes = plan.total();
  return HELIX_OK;
}

}  // extern "C"

namespace helix {
namespace {

// The partial attention of requests [b_begin, b_end); with o_out non-null (GQA only) the kernel
// also merges the shards of every KV-head group into o_out / lse_out (fused combine).
// Every check of a partial call except those on the workspace; fills the launch plan.
helix_status check_partial(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                           float softmax_scale, int32_t b_begin, int32_t b_end,
                           const float* o_partial, const float* lse, const void* o_out,
                           int32_t o_dtype, const float* lse_out, PartialPlan* plan) {
  if (c == nullptr || b_begin < 0 || b_end < b_begin || b_end > c->batch)
    return HELIX_ERR_INVALID_ARG;
  helix_status st = plan_partial(c, num_q_heads, plan);
  if (st != HELIX_OK) return st;
  if (q == nullptr || o_partial == nullptr || lse == nullptr) return HELIX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o_partial) || !aligned4(lse)) return HELIX_ERR_INVALID_ARG;
  if (o_out != nullptr && (c->kind != HELIX_ATTN_GQA || (o_dtype != 0 && o_dtype != 1) ||
                           !aligned16(o_out) || !aligned4(lse_out)))
    return HELIX_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return HELIX_ERR_INVALID_ARG;
  return HELIX_OK;
}

helix_status partial_impl(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                          float softmax_scale, int32_t b_begin, int32_t b_end, float* o_partial,
                          float* lse, void* workspace, size_t workspace_bytes, void* o_out,
                          int32_t o_dtype, float* lse_out, cudaStream_t stream) {
  PartialPlan plan;
  helix_status st = check_partial(c, q, num_q_heads, softmax_scale, b_begin, b_end, o_partial,
                                  lse, o_out, o_dtype, lse_out, &plan);
  if (st != HELIX_OK) return st;
  if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < plan.total())
    return HELIX_ERR_INVALID_ARG;
  if (b_end == b_begin) return HELIX_OK;
  // units are ordered request-major, so a request range is a contiguous unit range
  const int units_per_request = plan.units / c->batch;
  const int u0 = b_begin * units_per_request;
  const int units = (b_end - b_begin) * units_per_request;

  if (c->kind == HELIX_ATTN_MLA) {
    MlaParams m{};
    m.page_table = c->page_table;
    m.shard_lens = c->shard_lens;
    m.o_part = o_partial;
    m.lse = lse;
    m.pool = static_cast<const uint8_t*>(c->k_pool);
    m.tickets = reinterpret_cast<int32_t*>(workspace);
    m.seg = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + plan.ticket_bytes +
                                     plan.gticket_bytes);
    m.err = c->err_word;
    m.B = c->batch;
    m.kvp = c->kvp;
    m.max_pages = c->max_pages_per_shard;
    m.num_pages = c->num_pages;
    m.scale_log2 = softmax_scale * 1.4426950408889634f;
    // latent pool as [9 chunks][pages * 64 rows][64 columns]: boxes of two chunks of a page (a
    // score slot, or a value slot of 128 columns); q as [B * 128][576], boxes of 64 columns x 64
    // rows (one CTA's heads); 128-byte swizzle for the tensor-core operand layout
    CUtensorMap tmC, tmQ;
    if (!encode_latent_chunks_map(&tmC, c->k_pool, (uint64_t)c->num_pages * 64) ||
        !encode_rows_map(&tmQ, const_cast<void*>(q), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 576,
                         (uint64_t)c->batch * 128, 64, 64))
      return HELIX_ERR_CUDA;
    // request ranges of at most plan.max_units units each, one after another on the stream
    // (they share the workspace; the unit tickets are back at zero after each launch)
    const int per = plan.max_units / units_per_request;
    for (int b = b_begin; b < b_end; b += per) {
      m.u0 = b * units_per_request;
      m.units = (min(b_end, b + per) - b) * units_per_request;
      st = mla_partial_launch(tmC, tmQ, m, plan.grid, stream);
      if (st != HELIX_OK) return st;
    }
    return HELIX_OK;
  }

  GqaParams p{};
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  p.page_table = c->page_table;
  p.shard_lens = c->shard_lens;
  p.o_part = o_partial;
  p.lse = lse;
  p.tickets = reinterpret_cast<int32_t*>(workspace);
  p.gtickets =
      reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(workspace) + plan.ticket_bytes);
  p.seg = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + plan.ticket_bytes +
                                   plan.gticket_bytes);
  p.o_out = o_out;
  p.o_dtype = o_dtype;
  p.lse_out = o_out != nullptr ? lse_out : nullptr;
  p.err = c->err_word;
  p.B = c->batch;
  p.Hq = num_q_heads;
  p.Hkv = c->num_kv_heads;
  p.G = num_q_heads / c->num_kv_heads;
  p.D = c->head_dim;
  p.kvp = c->kvp;
  p.max_pages = c->max_pages_per_shard;
  p.num_pages = c->num_pages;
  p.units = units;
  p.u0 = u0;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  if (c->kv_dtype == HELIX_KV_NVFP4) {
    p.k_codes = reinterpret_cast<const uint8_t*>(c->k_pool);
    p.k_scale = reinterpret_cast<const uint8_t*>(c->k_scale);
    p.v_codes = reinterpret_cast<const uint8_t*>(c->v_pool);
    p.v_scale = reinterpret_cast<const uint8_t*>(c->v_scale);
    return gqa_partial_nvfp4_launch(p, plan.grid, stream);
  }

  const uint64_t rows = (uint64_t)c->num_pages * c->num_kv_heads * c->page_tokens;
  CUtensorMap tmK, tmV;
  if (!encode_rows_map(&tmK, c->k_pool, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c->head_dim, rows,
                       64, 64) ||
      !encode_rows_map(&tmV, c->v_pool, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c->head_dim, rows,
                       64, 64))
    return HELIX_ERR_CUDA;
  return gqa_partial_bf16_launch(tmK, tmV, p, plan.grid, stream);
}

}  // namespace

helix_status validate_partial_call(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                                   float softmax_scale, const float* o_partial, const float* lse,
                                   size_t* workspace_bytes) {
  PartialPlan plan;
  helix_status st = check_partial(c, q, num_q_heads, softmax_scale, 0, c ? c->batch : 0,
                                  o_partial, lse, nullptr, 0, nullptr, &plan);
  if (st != HELIX_OK) return st;
  *workspace_bytes = plan.total();
  return HELIX_OK;
}

}  // namespace helix

extern "C" {

helix_status helix_stream_wait(helix_stream_t stream, helix_event_t event, uint64_t limit_us) {
  if (event == nullptr) return HELIX_ERR_INVALID_ARG;
  auto ev = reinterpret_cast<cudaEvent_t>(event);
  if (cudaEventRecord(ev, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HELIX_ERR_CUDA;
  return poll_with_limit(
      [ev]() {
        const cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return PollResult::kDone;
        if (e == cudaErrorNotReady) {
          // a pending query is not an error: if the runtime recorded it as the last error, clear
          // it so that a later launch check does not read it as a failure
          if (cudaPeekAtLastError() == cudaErrorNotReady) (void)cudaGetLastError();
          return PollResult::kPending;
        }
        return PollResult::kError;
      },
      limit_us);
}

helix_status helix_attn_partial_range(const helix_kv_cache* c, const void* q,
                                      int32_t num_q_heads, float softmax_scale, int32_t b_begin,
                                      int32_t b_end, float* o_partial, float* lse, void* workspace,
                                      size_t workspace_bytes, helix_stream_t stream) {
  return partial_impl(c, q, num_q_heads, softmax_scale, b_begin, b_end, o_partial, lse, workspace,
                      workspace_bytes, nullptr, 0, nullptr,
                      reinterpret_cast<cudaStream_t>(stream));
}

helix_status helix_attn_partial_combine(const helix_kv_cache* c, const void* q,
                                        int32_t num_q_heads, float softmax_scale,
                                        float* o_partial, float* lse, void* o_out,
                                        int32_t o_dtype, float* lse_out, void* workspace,
                                        size_t workspace_bytes, helix_stream_t stream) {
  if (c == nullptr) return HELIX_ERR_INVALID_ARG;
  if (c->kind == HELIX_ATTN_GQA)
    return partial_impl(c, q, num_q_heads, softmax_scale, 0, c->batch, o_partial, lse, workspace,
                        workspace_bytes, o_out, o_dtype, lse_out,
                        reinterpret_cast<cudaStream_t>(stream));
  // MLA: a whole request's 128 x 512 merge is too large for one CTA; two launches
  if (o_out == nullptr || (o_dtype != 0 && o_dtype != 1) || !aligned16(o_out) ||
      !aligned4(lse_out))
    return HELIX_ERR_INVALID_ARG;
  helix_status st = partial_impl(c, q, num_q_heads, softmax_scale, 0, c->batch, o_partial, lse,
                                 workspace, workspace_bytes, nullptr, 0, nullptr,
                                 reinterpret_cast<cudaStream_t>(stream));
  if (st != HELIX_OK) return st;
  return helix_attn_combine(c->kvp, c->batch, num_q_heads, c->v_dim, o_partial, lse, o_out,
                            o_dtype, lse_out, stream);
}

helix_status helix_attn_partial(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                                float softmax_scale, float* o_partial, float* lse, void* workspace,
                                size_t workspace_bytes, helix_stream_t stream) {
  if (c == nullptr) return HELIX_ERR_INVALID_ARG;
  return helix_attn_partial_range(c, q, num_q_heads, softmax_scale, 0, c->batch, o_partial, lse,
                                  workspace, workspace_bytes, stream);
}

helix_status helix_attn_combine_range(int32_t kvp, int32_t batch, int32_t num_q_heads,
                                      int32_t v_dim, int32_t b_begin, int32_t b_end,
                                      const float* o_partial, const float* lse, void* o_out,
                                      int32_t o_dtype, float* lse_out, helix_stream_t stream) {
  if (kvp < 1 || batch < 0 || num_q_heads < 0 || v_dim < 4 || v_dim % 4 != 0)
    return HELIX_ERR_INVALID_ARG;
  if (b_begin < 0 || b_end < b_begin || b_end > batch) return HELIX_ERR_INVALID_ARG;
  if (o_dtype != 0 && o_dtype != 1) return HELIX_ERR_INVALID_ARG;
  if (o_partial == nullptr || lse == nullptr || o_out == nullptr) return HELIX_ERR_INVALID_ARG;
  if (!aligned16(o_partial) || !aligned4(lse) || !aligned16(o_out) || !aligned4(lse_out))
    return HELIX_ERR_INVALID_ARG;
  return combine_launch(kvp, batch * num_q_heads, b_begin * num_q_heads,
                        (b_end - b_begin) * num_q_heads, v_dim, o_partial, lse, o_out, o_dtype,
                        lse_out, reinterpret_cast<cudaStream_t>(stream));
}

helix_status helix_attn_combine(int32_t kvp, int32_t batch, int32_t num_q_heads, int32_t v_dim,
                                const float* o_partial, const float* lse, void* o_out,
                                int32_t o_dtype, float* lse_out, helix_stream_t stream) {
  return helix_attn_combine_range(kvp, batch, num_q_heads, v_dim, 0, batch, o_partial, lse, o_out,
                                  o_dtype, lse_out, stream);
}

helix_status helix_attn_combine_sources(int32_t nsrc, const float* const* o_parts,
                                        const float* const* lses, int32_t batch,
                                        int32_t num_q_heads, int32_t v_dim, int32_t head_begin,
                                        int32_t head_end, void* o_out, int32_t o_dtype,
                                        float* lse_out, helix_stream_t stream) {
  if (nsrc < 1 || nsrc > HELIX_MAX_SOURCES || o_parts == nullptr || lses == nullptr)
    return HELIX_ERR_INVALID_ARG;
  if (batch < 1 || num_q_heads < 1 || v_dim < 4 || v_dim % 4 != 0 || head_begin < 0 ||
      head_end <= head_begin || head_end > num_q_heads)
    return HELIX_ERR_INVALID_ARG;
  if (o_out == nullptr || (o_dtype != 0 && o_dtype != 1) || !aligned16(o_out) ||
      !aligned4(lse_out))
    return HELIX_ERR_INVALID_ARG;
  if ((int64_t)batch * num_q_heads * v_dim > INT32_MAX) return HELIX_ERR_CAPACITY;
  CombineSources src{};
  src.n = nsrc;
  for (int s = 0; s < nsrc; ++s) {
    if (o_parts[s] == nullptr || lses[s] == nullptr || !aligned16(o_parts[s]) ||
        !aligned4(lses[s]))
      return HELIX_ERR_INVALID_ARG;
    src.o[s] = o_parts[s];
    src.lse[s] = lses[s];
  }
  return combine_sources_launch(src, batch, num_q_heads, head_begin, head_end - head_begin, v_dim,
                                o_out, o_dtype, lse_out, static_cast<cudaStream_t>(stream));
}

helix_status helix_attn_overlapped(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                                   float softmax_scale, int32_t n_groups, float* o_partial,
                                   float* lse, void* o_out, int32_t o_dtype, float* lse_out,
                                   void* workspace, size_t workspace_bytes,
                                   helix_stream_t stream_a, helix_stream_t stream_b,
                                   const helix_event_t* events) {
  if (c == nullptr || events == nullptr || n_groups < 1) return HELIX_ERR_INVALID_ARG;
  if (stream_a == stream_b) return HELIX_ERR_INVALID_ARG;
  for (int g = 0; g <= n_groups; ++g)
    if (events[g] == nullptr) return HELIX_ERR_INVALID_ARG;
  // validate everything before the first launch, so an error launches nothing
  PartialPlan plan;
  helix_status st = plan_partial(c, num_q_heads, &plan);
  if (st != HELIX_OK) return st;
  if (q == nullptr || o_partial == nullptr || lse == nullptr || workspace == nullptr ||
      o_out == nullptr || (o_dtype != 0 && o_dtype != 1) || c->v_dim % 4 != 0)
    return HELIX_ERR_INVALID_ARG;
  if (!aligned16(o_out) || !aligned4(lse_out)) return HELIX_ERR_INVALID_ARG;
  const int B = c->batch;
  const int groups = n_groups < B ? n_groups : B;
  const int per = (B + groups - 1) / groups;
  auto sa = reinterpret_cast<cudaStream_t>(stream_a);
  auto sb = reinterpret_cast<cudaStream_t>(stream_b);
  for (int g = 0; g * per < B; ++g) {
    const int b0 = g * per, b1 = b0 + per < B ? b0 + per : B;
    // stream A: partial attention of request group g (groups run back to back on A, sharing the
    // workspace); stream B: combine of group g once its partials exist, overlapping group g+1
    st = helix_attn_partial_range(c, q, num_q_heads, softmax_scale, b0, b1, o_partial, lse,
                                  workspace, workspace_bytes, stream_a);
    if (st != HELIX_OK) return st;
    auto ev = reinterpret_cast<cudaEvent_t>(events[g]);
    if (cudaEventRecord(ev, sa) != cudaSuccess || cudaStreamWaitEvent(sb, ev, 0) != cudaSuccess)
      return HELIX_ERR_CUDA;
    st = helix_attn_combine_range(c->kvp, B, num_q_heads, c->v_dim, b0, b1, o_partial, lse, o_out,
                                  o_dtype, lse_out, stream_b);
    if (st != HELIX_OK) return st;
  }
  // join: stream A waits for the last combine, so the caller needs to order only against A
  auto done = reinterpret_cast<cudaEvent_t>(events[n_groups]);
  if (cudaEventRecord(done, sb) != cudaSuccess || cudaStreamWaitEvent(sa, done, 0) != cudaSuccess)
    return HELIX_ERR_CUDA;
  return HELIX_OK;
}

helix_status helix_decode_overlapped(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                                    float softmax_scale, int32_t n_groups, const void* k_new,
                                    const void* v_new, const void* k_new_scale,
                                    const void* v_new_scale, int32_t n_new,
                                    const int32_t* group_n_valid, float* o_partial, float* lse,
                                    void* o_out, int32_t o_dtype, float* lse_out, void* workspace,
                                    size_t workspace_bytes, helix_stream_t stream_a,
                                    helix_stream_t stream_b, const helix_event_t* events) {
  if (c == nullptr || events == nullptr || n_groups < 1 || group_n_valid == nullptr)
    return HELIX_ERR_INVALID_ARG;
  if (stream_a == stream_b || n_new < 1) return HELIX_ERR_INVALID_ARG;
  const int B = c->batch;
  const int groups = n_groups < B ? n_groups : B;
  for (int e = 0; e < 2 * groups + 1; ++e)
    if (events[e] == nullptr) return HELIX_ERR_INVALID_ARG;
  PartialPlan plan;
  helix_status st = plan_partial(c, num_q_heads, &plan);
  if (st != HELIX_OK) return st;
  if (q == nullptr || o_partial == nullptr || lse == nullptr || workspace == nullptr ||
      o_out == nullptr || (o_dtype != 0 && o_dtype != 1) || c->v_dim % 4 != 0 ||
      !aligned16(o_out) || !aligned4(lse_out) || !aligned4(group_n_valid))
    return HELIX_ERR_INVALID_ARG;
  const int per = (B + groups - 1) / groups;
  const int ng = (B + per - 1) / per;  // groups actually formed
  auto sa = reinterpret_cast<cudaStream_t>(stream_a);
  auto sb = reinterpret_cast<cudaStream_t>(stream_b);
  auto ev_app = [&](int g) { return reinterpret_cast<cudaEvent_t>(events[g]); };
  auto ev_part = [&](int g) { return reinterpret_cast<cudaEvent_t>(events[groups + g]); };
  auto append_group = [&](int g) -> helix_status {  // on stream B; row g of group_n_valid
    helix_status s2 = helix_kv_append(c, k_new, v_new, k_new_scale, v_new_scale, n_new,
                                      group_n_valid + (size_t)g * B, stream_b);
    if (s2 != HELIX_OK) return s2;
    return cudaEventRecord(ev_app(g), sb) == cudaSuccess ? HELIX_OK : HELIX_ERR_CUDA;
  };
  st = append_group(0);
  if (st != HELIX_OK) return st;
  for (int g = 0; g < ng; ++g) {
    const int b0 = g * per, b1 = b0 + per < B ? b0 + per : B;
    // stream A: group g's partial once its new tokens are in the cache
    if (cudaStreamWaitEvent(sa, ev_app(g), 0) != cudaSuccess) return HELIX_ERR_CUDA;
    st = helix_attn_partial_range(c, q, num_q_heads, softmax_scale, b0, b1, o_partial, lse,
                                  workspace, workspace_bytes, stream_a);
    if (st != HELIX_OK) return st;
    if (cudaEventRecord(ev_part(g), sa) != cudaSuccess) return HELIX_ERR_CUDA;
    // stream B: the next group's append overlaps this partial, then this group's combine
    if (g + 1 < ng) {
      st = append_group(g + 1);
      if (st != HELIX_OK) return st;
    }
    if (cudaStreamWaitEvent(sb, ev_part(g), 0) != cudaSuccess) return HELIX_ERR_CUDA;
    st = helix_attn_combine_range(c->kvp, B, num_q_heads, c->v_dim, b0, b1, o_partial, lse, o_out,
                                  o_dtype, lse_out, stream_b);
    if (st != HELIX_OK) return st;
  }
  auto done = reinterpret_cast<cudaEvent_t>(events[2 * groups]);
  if (cudaEventRecord(done, sb) != cudaSuccess || cudaStreamWaitEvent(sa, done, 0) != cudaSuccess)
    return HELIX_ERR_CUDA;
  return HELIX_OK;
}

}  // extern "C"
