// internal.h -- host-side declarations shared by the helix translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "helix.h"

namespace helix {

// Parameters of the GQA partial kernels (bf16 and NVFP4 KV).
struct GqaParams {
  const __nv_bfloat16* q;     // [B][Hq][D]
  const int32_t* page_table;  // [kvp][B][max_pages]
  const int32_t* shard_lens;  // [kvp][B]
  float* o_part;              // [kvp][B][Hq][D]
  float* lse;                 // [kvp][B][Hq]
  int32_t* tickets;           // [units], zero between launches
  float* seg;                 // [grid][2][record]
  uint32_t* err;              // may be null
  const uint8_t* k_scale;     // NVFP4 only: [pages][Hkv][64][D/16]
  const uint8_t* v_scale;
  const uint8_t* k_codes;     // NVFP4 only: [pages][Hkv][64][D/2]
  const uint8_t* v_codes;
  int B, Hq, Hkv, G, D, kvp, max_pages, num_pages, units;
  int u0;                     // first unit of this launch (a request boundary)
  float scale_log2;  // softmax_scale * log2(e)
  // fused combine (o_out non-null): the CTA that finishes the last of the kvp units of a group
  // (b, k) merges the group's rows into o_out / lse_out
  void* o_out;                // [B][Hq][D], bf16 (o_dtype 0) or fp32 (1)
  float* lse_out;             // [B][Hq], may be null
  int32_t* gtickets;          // [B * Hkv], zero between launches
  int o_dtype;
};

size_t gqa_partial_smem_bytes(int head_dim, int units);  // bf16 kernel
size_t gqa_segment_record_floats(int head_dim);
size_t gqa_nvfp4_smem_bytes(int units);                  // NVFP4 kernel (head_dim 128)
size_t gqa_nvfp4_segment_record_floats();
helix_status gqa_partial_bf16_launch(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                     const GqaParams& p, int grid, cudaStream_t stream);
helix_status gqa_partial_nvfp4_launch(const GqaParams& p, int grid, cudaStream_t stream);

// Parameters of the MLA partial kernel (128 heads, one 576-wide latent head, values = first 512).
struct MlaParams {
  const int32_t* page_table;  // [kvp][B][max_pages]
  const int32_t* shard_lens;  // [kvp][B]
  float* o_part;              // [kvp][B][128][512]
  float* lse;                 // [kvp][B][128]
  const uint8_t* pool;        // bf16 [pages * 64][576] (also read through the tensor maps)
  int32_t* tickets;           // [units][2], zero between launches
  float* seg;                 // [clusters][2 slots][2 CTAs][record]
  uint32_t* err;              // may be null
  int B, kvp, max_pages, num_pages, units;
  int u0;                     // first unit of this launch (a request boundary)
  float scale_log2;
};
size_t mla_partial_smem_bytes(int units);
size_t mla_segment_record_floats();
helix_status mla_partial_launch(const CUtensorMap& tmC, const CUtensorMap& tmQ,
                                const MlaParams& p, int grid, cudaStream_t stream);

// Append: copies the new tokens' rows (and scales) into their pages.
struct AppendParams {
  const uint8_t* src[4];   // k rows, v rows, k scales, v scales (null when unused)
  uint8_t* dst[4];         // matching pools
  int row_bytes[4];        // bytes per (token, head) row of each stream; 0 = unused
  const int32_t* page_table;
  int32_t* shard_lens;
  int32_t* seq_lens;
  uint32_t* err;
  const int32_t* n_valid;  // optional [B]
  int v_nvfp4;             // 1: streams 1 and 3 (V codes, V scales) use the token-pair layout
  int quantize;            // 1: src[0] / src[1] are bf16 K / V rows of d = 128, encoded to NVFP4
                           //    on the device into the four NVFP4 pools (dst[0..3])
  int B, Hkv, kvp, layout, rr_block, contig_chunk, page_tokens, max_pages, num_pages, n_new;
};
helix_status append_launch(const AppendParams& p, cudaStream_t stream);

// Every host-side check of helix_attn_partial over the whole batch except those on the workspace
// (launches nothing); on success *workspace_bytes is the scratch the call needs.
helix_status validate_partial_call(const helix_kv_cache* c, const void* q, int32_t num_q_heads,
                                   float softmax_scale, const float* o_partial, const float* lse,
                                   size_t* workspace_bytes);

// Raises a kernel's dynamic shared-memory limit to the device maximum, once per (kernel, device).
cudaError_t allow_max_dynamic_smem(const void* func);

// rows = B * Hq (the shard stride of o_partial / lse); combines rows [row0, row0 + nrows)
// Sources of a combine over separate buffers: source s holds O [B][Hq][v_dim] at o[s] and lse
// [B][Hq] at lse[s] (device-accessible; on a multi-GPU node, peer mappings of other GPUs' buffers).
struct CombineSources {
  int n;
  const float* o[HELIX_MAX_SOURCES];
  const float* lse[HELIX_MAX_SOURCES];
};
helix_status combine_sources_launch(const CombineSources& src, int B, int Hq, int h0, int nh,
                                    int v_dim, void* o_out, int o_dtype, float* lse_out,
                                    cudaStream_t stream);
helix_status combine_launch(int kvp, int rows, int row0, int nrows, int v_dim,
                            const float* o_partial, const float* lse, void* o_out, int o_dtype,
                            float* lse_out, cudaStream_t stream);

}  // namespace helix
