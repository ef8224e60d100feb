// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/paged_kv.h"

namespace pkv {

// Number of pkv_kv_dtype values.
constexpr int kNumKvFormats = 4;

// KV formats of the pools (pkv_kv_dtype).
// One-byte element codes (E4M3, INT8)?
__host__ __device__ constexpr bool k8(int fmt) {
  return fmt == PKV_KV_FP8_E4M3 || fmt == PKV_KV_INT8;
}
// FP4: E2M1 code pairs plus E4M3 block scales?
__host__ __device__ constexpr bool fp4(int fmt) { return fmt == PKV_KV_NVFP4; }
// Quantised, with per-(page, kv head) scales (every format but bf16)?
__host__ __device__ constexpr bool quant(int fmt) { return fmt != PKV_KV_BF16; }

// Bytes of one token row of one kv head in a pool: element codes, and the
// FP4 block scales (stored after every row's codes).
__host__ __device__ constexpr int row_code_bytes(int fmt, int head_dim) {
  return fmt == PKV_KV_BF16 ? 2 * head_dim : fp4(fmt) ? head_dim / 2 : head_dim;
}
__host__ __device__ constexpr int row_scale_bytes(int fmt, int head_dim) {
  return fp4(fmt) ? head_dim / 16 : 0;
}

struct AppendParams {
  uint8_t* k_pool;
  uint8_t* v_pool;
  uint8_t* k_blocks;  // FP4: block scales of the K pool (after its codes); else null
  uint8_t* v_blocks;
  const float* k_scale;
  const float* v_scale;
  const int32_t* page_table;
  const int32_t* seq_lens_before;
  const int32_t* cu_new;
  const uint4* k_new;  // [T][Hkv][D] bf16, as 16-byte vectors
  const uint4* v_new;
  int32_t* flags;
  int32_t batch;
  int32_t total_new;
  int32_t max_pages;
  int32_t num_pages;
  int32_t page_size;
  int32_t num_kv_heads;
  int32_t head_dim;
};

struct DecodeParams {
  const __nv_bfloat16* q;  // [B][Hq][D]
  const int32_t* page_table;
  const int32_t* seq_lens;
  const float* k_scale;  // [pages][Hkv] (E4M3)
  const float* v_scale;
  __nv_bfloat16* out;  // [B][Hq][D]
  float* lse;          // [B][Hq] or null
  float* part_o;       // [U + C][G][D]
  float2* part_ml;     // [U + C][G]
  int2* unit_info;     // [U]: (first partial slot, number of segments)
  int32_t* flags;
  // Fused append (all null otherwise): one new token per sequence, at
  // position seq_lens[b] - 1, written into the pools before it is read.
  const __nv_bfloat16* k_new;  // [B][Hkv][D]
  const __nv_bfloat16* v_new;
  uint8_t* k_pool;
  uint8_t* v_pool;
  uint8_t* k_blocks_w;  // FP4 fused append: block-scale regions to write
  uint8_t* v_blocks_w;
  // FP4 pools: the block-scale regions (after the codes) that the loads read
  const uint8_t* k_blocks;
  const uint8_t* v_blocks;
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t group;
  int32_t max_pages;
  int32_t num_pages;
  int32_t page_size;
  float scale_log2;  // softmax_scale * log2(e)
};

// fmt: the pool's pkv_kv_dtype
cudaError_t launch_append(const AppendParams& p, int fmt, int num_sms, cudaStream_t stream);
cudaError_t decode_occupancy(int head_dim, int fmt, int group, int* ctas_per_sm);
cudaError_t decode_run(int head_dim, int fmt, const CUtensorMap& tk, const CUtensorMap& tv,
                       const DecodeParams& p, int num_ctas, cudaStream_t stream);

cudaError_t launch_combine(const void* parts, const float* lse_parts, int num_parts, int rows,
                           int head_dim, void* out, float* lse, cudaStream_t stream);

int check_cache(const pkv_cache* c);
int check_group(const pkv_cache* c, int32_t num_q_heads, int32_t gqa_group);
int check_table_span(const pkv_cache* c, int32_t max_pages_per_seq);
int64_t block_region_offset(const pkv_cache* c);
int encode_pool_map(CUtensorMap* map, void* base, bool bytes, int64_t rows, int row_elems,
                    int box_cols, int box_rows);
int prefill_entry(const pkv_cache* cache, const void* q, int32_t num_q_heads, int32_t gqa_group,
                  const int32_t* cu_q_lens, const int32_t* page_table, int32_t max_pages_per_seq,
                  const int32_t* seq_lens, int32_t num_chunks, int32_t total_q,
                  int32_t max_q_len, float softmax_scale, void* out, float* lse,
                  cudaStream_t stream);

}  // namespace pkv
