// C ABI of libpagedkv.so (declared in include/paged_kv.h).
//
// Host side only: argument validation (every error is returned before any
// launch), decode planning, TMA tensor-map encoding and kernel launches.
// All device memory belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace pkv {

// ------------------------------------------------------------- utilities
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PKV_ERR_CUDA;
  return PKV_OK;
}

// Byte offset of an FP4 pool's block-scale region: all rows' codes come first.
int64_t block_region_offset(const pkv_cache* c) {
  return (int64_t)c->num_pages * c->num_kv_heads * c->page_size * (c->head_dim / 2);
}

// Validation shared by every entry point that reads the cache.
int check_cache(const pkv_cache* c) {
  if (!c) return PKV_ERR_NULL;
  if (!c->k_pool || !c->v_pool) return PKV_ERR_NULL;
  if (!aligned16(c->k_pool) || !aligned16(c->v_pool)) return PKV_ERR_ALIGN;
  if (c->num_pages < 1 || c->num_kv_heads < 1) return PKV_ERR_SHAPE;
  if (c->page_size != 64 && c->page_size != 128) return PKV_ERR_PAGE_SIZE;
  if (c->head_dim != 64 && c->head_dim != 128) return PKV_ERR_HEAD_DIM;
  if (c->kv_dtype != PKV_KV_BF16 && c->kv_dtype != PKV_KV_FP8_E4M3 &&
      c->kv_dtype != PKV_KV_INT8 && c->kv_dtype != PKV_KV_NVFP4)
    return PKV_ERR_DTYPE;
  if (c->kv_dtype != PKV_KV_BF16 && (!c->k_scale || !c->v_scale)) return PKV_ERR_DTYPE;
  // pool rows (pages * heads * page_size) index a TMA tensor: keep them in int32
  const long long rows = (long long)c->num_pages * c->num_kv_heads * c->page_size;
  if (rows >= INT_MAX) return PKV_ERR_SHAPE;
  return PKV_OK;
}

// Tokens a page-table row can address, max_pages_per_seq * page_size, must
// fit in int32: the kernels compare lengths against it in 32-bit arithmetic.
int check_table_span(const pkv_cache* c, int32_t max_pages_per_seq) {
  if ((int64_t)max_pages_per_seq * c->page_size > INT32_MAX) return PKV_ERR_SHAPE;
  return PKV_OK;
}

int check_group(const pkv_cache* c, int32_t num_q_heads, int32_t gqa_group) {
  if (gqa_group != 1 && gqa_group != 2 && gqa_group != 4 && gqa_group != 8) return PKV_ERR_GQA;
  if (num_q_heads != gqa_group * c->num_kv_heads) return PKV_ERR_GQA;
  return PKV_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D view [rows][row_elems] of a pool's codes (bytes, or bf16 elements)
// with a [box_rows][box_cols] box and the swizzle of the box's row width
// (128, 64 or 32 bytes).
int encode_pool_map(CUtensorMap* map, void* base, bool bytes, int64_t rows, int row_elems,
                    int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PKV_ERR_CUDA;
  const int eb = bytes ? 1 : 2;
  const int box_bytes = box_cols * eb;
  cuuint64_t dims[2] = {(cuuint64_t)row_elems, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_elems * eb};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw = box_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

static int decode_ctas_per_sm(int head_dim, int fmt, int group, int* out) {
  // Cached per device and variant: a kernel's occupancy does not change at
  // run time, but the shared-memory attribute that decode_occupancy sets
  // belongs to the device that is current, so every device fills its own
  // entry (and sets its own attribute) on first use.
  constexpr int kMaxDevices = 64;
  static int cache[kMaxDevices][2][kNumKvFormats][4] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices || fmt < 0 || fmt >= kNumKvFormats) return PKV_ERR_UNSUPPORTED;
  const int gi = group == 1 ? 0 : group == 2 ? 1 : group == 4 ? 2 : 3;
  std::lock_guard<std::mutex> lock(mu);
  int& slot = cache[dev][head_dim == 128][fmt][gi];
  if (slot == 0) {
    int n = 0;
    if (decode_occupancy(head_dim, fmt, group, &n) != cudaSuccess || n < 1) return PKV_ERR_CUDA;
    slot = n;
  }
  *out = slot;
  return PKV_OK;
}

// Upper bound of decode CTAs used for workspace sizing.
constexpr int kMaxDecodeCtasPerSm = 4;

}  // namespace pkv

using namespace pkv;

extern "C" {

int pkv_abi_version(void) { return (1 << 16) | 1; }

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL: return "a required pointer is NULL";
    case PKV_ERR_SHAPE: return "a count or size is negative or inconsistent";
    case PKV_ERR_PAGE_SIZE: return "page_size must be 64 or 128";
    case PKV_ERR_HEAD_DIM: return "head_dim must be 64 or 128";
    case PKV_ERR_GQA: return "num_q_heads must equal gqa_group * num_kv_heads, group in {1,2,4,8}";
    case PKV_ERR_DTYPE: return "unknown kv dtype, or E4M3 pools without scales";
    case PKV_ERR_WORKSPACE: return "decode workspace is NULL, misaligned or too small";
    case PKV_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case PKV_ERR_ALIGN: return "a pointer that must be 16-byte aligned is not";
    case PKV_ERR_UNSUPPORTED: return "this combination is not implemented";
    case PKV_ERR_SCRATCH_LIMIT:
      return "the request needs more decode scratch than the library's static 16 MiB array";
    case PKV_ERR_NO_PAGES: return "the free pages cannot cover the growth request";
    default: return "unknown status";
  }
}

int paged_kv_append(const pkv_cache* cache, const int32_t* page_table, int32_t max_pages_per_seq,
                    const int32_t* seq_lens_before, const int32_t* cu_new_tokens, int32_t batch,
                    int32_t total_new_tokens, const void* k_new, const void* v_new,
                    void* stream) {
  int st = check_cache(cache);
  if (st) return st;
  if (batch < 0 || total_new_tokens < 0 || max_pages_per_seq < 1) return PKV_ERR_SHAPE;
  if ((st = check_table_span(cache, max_pages_per_seq))) return st;
  if (total_new_tokens == 0 || batch == 0) return PKV_OK;
  if (!page_table || !seq_lens_before || !cu_new_tokens || !k_new || !v_new) return PKV_ERR_NULL;
  if (!aligned16(k_new) || !aligned16(v_new)) return PKV_ERR_ALIGN;
  int sms = 0;
  if ((st = device_sms(&sms))) return st;
  AppendParams p;
  p.k_pool = static_cast<uint8_t*>(cache->k_pool);
  p.v_pool = static_cast<uint8_t*>(cache->v_pool);
  p.k_blocks = fp4(cache->kv_dtype) ? p.k_pool + block_region_offset(cache) : nullptr;
  p.v_blocks = fp4(cache->kv_dtype) ? p.v_pool + block_region_offset(cache) : nullptr;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  p.page_table = page_table;
  p.seq_lens_before = seq_lens_before;
  p.cu_new = cu_new_tokens;
  p.k_new = static_cast<const uint4*>(k_new);
  p.v_new = static_cast<const uint4*>(v_new);
  p.flags = cache->error_flags;
  p.batch = batch;
  p.total_new = total_new_tokens;
  p.max_pages = max_pages_per_seq;
  p.num_pages = cache->num_pages;
  p.page_size = cache->page_size;
  p.num_kv_heads = cache->num_kv_heads;
  p.head_dim = cache->head_dim;
  cudaError_t e = launch_append(p, cache->kv_dtype, sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int paged_decode_plan(int32_t batch, int32_t num_kv_heads, int32_t max_seq_len,
                      int32_t num_sms, int32_t num_ctas, int32_t ctas_per_sm,
                      int32_t* out_ctas) {
  if (!out_ctas) return PKV_ERR_NULL;
  if (batch < 0 || num_kv_heads < 1 || max_seq_len < 0 || num_sms < 1 || num_ctas < 0 ||
      ctas_per_sm < 1)
    return PKV_ERR_SHAPE;
  // 64-token work-list tiles of the largest possible batch (an upper bound on
  // the tiles of every format; the kernel lets only min(C, T) CTAs work).
  const long long max_tiles = (long long)batch * num_kv_heads * ((max_seq_len + 63) / 64);
  long long c = num_ctas > 0 ? num_ctas : (long long)num_sms * ctas_per_sm;
  if (c > max_tiles) c = max_tiles;
  if (c < 1) c = 1;
  *out_ctas = (int32_t)c;
  return PKV_OK;
}

size_t paged_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t max_seq_len, int32_t num_ctas) {
  if (batch < 0 || num_kv_heads < 1 || num_q_heads < num_kv_heads || head_dim < 1 ||
      max_seq_len < 0 || num_ctas < 0)
    return 0;
  int sms = 0;
  if (device_sms(&sms)) return 0;
  int32_t c = 0;
  if (paged_decode_plan(batch, num_kv_heads, max_seq_len, sms, num_ctas, kMaxDecodeCtasPerSm,
                        &c))
    return 0;
  const size_t G = (size_t)num_q_heads / num_kv_heads;
  const size_t units = (size_t)batch * num_kv_heads;
  const size_t slots = units + (size_t)c;
  size_t bytes = slots * G * head_dim * sizeof(float);  // partial o
  bytes = (bytes + 15) & ~size_t(15);
  bytes += slots * G * 2 * sizeof(float);  // partial (m, l)
  bytes = (bytes + 15) & ~size_t(15);
  bytes += units * sizeof(int2);  // per-unit (first slot, segments)
  return (bytes + 255) & ~size_t(255);
}

// Decode, with the fused append of one new token per sequence when k_new
// and v_new are given (both null otherwise).
static int decode_entry(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                        int32_t gqa_group, const int32_t* page_table, int32_t max_pages_per_seq,
                        const int32_t* seq_lens, int32_t batch, int32_t max_seq_len,
                        float softmax_scale, const void* k_new, const void* v_new, void* out,
                        float* lse, void* workspace, size_t workspace_bytes, int32_t num_ctas,
                        void* stream) {
  int st = check_cache(cache);
  if (st) return st;
  if ((st = check_group(cache, num_q_heads, gqa_group))) return st;
  if (batch < 0 || max_pages_per_seq < 1 || max_seq_len < 0 || num_ctas < 0) return PKV_ERR_SHAPE;
  if (!std::isfinite(softmax_scale)) return PKV_ERR_SHAPE;
  if (batch == 0) return PKV_OK;
  if (!q || !page_table || !seq_lens || !out) return PKV_ERR_NULL;
  if (!aligned16(q) || !aligned16(out)) return PKV_ERR_ALIGN;
  if ((st = check_table_span(cache, max_pages_per_seq))) return st;
  if ((int64_t)max_seq_len > (int64_t)max_pages_per_seq * cache->page_size) return PKV_ERR_SHAPE;
  const size_t need = paged_decode_workspace_bytes(batch, num_q_heads, cache->num_kv_heads,
                                                   cache->head_dim, max_seq_len, num_ctas);
  if (need == 0) return PKV_ERR_CUDA;
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return PKV_ERR_WORKSPACE;

  const int fmt = cache->kv_dtype;
  int sms = 0, per_sm = 0;
  if ((st = device_sms(&sms))) return st;
  if ((st = decode_ctas_per_sm(cache->head_dim, fmt, gqa_group, &per_sm))) return st;
  if (per_sm > kMaxDecodeCtasPerSm) per_sm = kMaxDecodeCtasPerSm;
  int32_t ctas = 0;
  if ((st = paged_decode_plan(batch, cache->num_kv_heads, max_seq_len, sms, num_ctas, per_sm,
                              &ctas)))
    return st;

  const int D = cache->head_dim;
  const int64_t rows = (int64_t)cache->num_pages * cache->num_kv_heads * cache->page_size;
  // quantised pools are viewed as bytes: a row holds D codes (one-byte
  // formats) or D/2 (FP4); bf16 rows are loaded in 64-element boxes
  const bool bytes = quant(fmt);
  const int row_elems = fp4(fmt) ? D / 2 : D;
  const int box_cols = bytes ? (row_elems >= 128 ? 128 : row_elems) : 64;
  CUtensorMap tk, tv;
  if ((st = encode_pool_map(&tk, cache->k_pool, bytes, rows, row_elems, box_cols, 64))) return st;
  if ((st = encode_pool_map(&tv, cache->v_pool, bytes, rows, row_elems, box_cols, 64))) return st;

  const size_t G = (size_t)gqa_group;
  const size_t units = (size_t)batch * cache->num_kv_heads;
  int32_t c_ws = 0;
  paged_decode_plan(batch, cache->num_kv_heads, max_seq_len, sms, num_ctas, kMaxDecodeCtasPerSm,
                    &c_ws);
  const size_t slots = units + (size_t)c_ws;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  size_t off = slots * G * D * sizeof(float);
  off = (off + 15) & ~size_t(15);
  float* part_o = reinterpret_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(ws + off);
  off += slots * G * 2 * sizeof(float);
  off = (off + 15) & ~size_t(15);
  int2* unit_info = reinterpret_cast<int2*>(ws + off);

  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.unit_info = unit_info;
  p.flags = cache->error_flags;
  if (fp4(fmt)) {
    p.k_blocks = static_cast<const uint8_t*>(cache->k_pool) + block_region_offset(cache);
    p.v_blocks = static_cast<const uint8_t*>(cache->v_pool) + block_region_offset(cache);
  }
  if (k_new) {
    p.k_new = static_cast<const __nv_bfloat16*>(k_new);
    p.v_new = static_cast<const __nv_bfloat16*>(v_new);
    p.k_pool = static_cast<uint8_t*>(cache->k_pool);
    p.v_pool = static_cast<uint8_t*>(cache->v_pool);
    if (fp4(fmt)) {
      p.k_blocks_w = p.k_pool + block_region_offset(cache);
      p.v_blocks_w = p.v_pool + block_region_offset(cache);
    }
  }
  p.batch = batch;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = cache->num_kv_heads;
  p.group = gqa_group;
  p.max_pages = max_pages_per_seq;
  p.num_pages = cache->num_pages;
  p.page_size = cache->page_size;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  cudaError_t e = decode_run(D, fmt, tk, tv, p, ctas, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int paged_decode_attention(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                           int32_t gqa_group, const int32_t* page_table,
                           int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t max_seq_len, float softmax_scale, void* out, float* lse,
                           void* workspace, size_t workspace_bytes, int32_t num_ctas,
                           void* stream) {
  return decode_entry(cache, q, num_q_heads, gqa_group, page_table, max_pages_per_seq, seq_lens,
                      batch, max_seq_len, softmax_scale, nullptr, nullptr, out, lse, workspace,
                      workspace_bytes, num_ctas, stream);
}

int paged_decode_attention_append(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                                  int32_t gqa_group, const int32_t* page_table,
                                  int32_t max_pages_per_seq, const int32_t* seq_lens,
                                  int32_t batch, int32_t max_seq_len, float softmax_scale,
                                  const void* k_new, const void* v_new, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, int32_t num_ctas,
                                  void* stream) {
  if (batch > 0 && (!k_new || !v_new)) return PKV_ERR_NULL;
  if (batch > 0 && (!aligned16(k_new) || !aligned16(v_new))) return PKV_ERR_ALIGN;
  return decode_entry(cache, q, num_q_heads, gqa_group, page_table, max_pages_per_seq, seq_lens,
                      batch, max_seq_len, softmax_scale, k_new, v_new, out, lse, workspace,
                      workspace_bytes, num_ctas, stream);
}

int paged_attention_combine(const void* parts, const float* lse_parts, int32_t num_parts,
                            int32_t rows, int32_t head_dim, void* out, float* lse,
                            void* stream) {
  if (num_parts < 1 || rows < 0) return PKV_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_HEAD_DIM;
  if (rows == 0) return PKV_OK;
  if (!parts || !lse_parts || !out) return PKV_ERR_NULL;
  if (!aligned16(parts) || !aligned16(out)) return PKV_ERR_ALIGN;
  if ((int64_t)num_parts * rows * head_dim >= INT64_C(1) << 40) return PKV_ERR_SHAPE;
  cudaError_t e = launch_combine(parts, lse_parts, num_parts, rows, head_dim, out, lse,
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int paged_prefill_chunk_attention(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                                  int32_t gqa_group, const int32_t* cu_q_lens,
                                  const int32_t* page_table, int32_t max_pages_per_seq,
                                  const int32_t* seq_lens, int32_t num_chunks, int32_t total_q,
                                  int32_t max_q_len, float softmax_scale, void* out, float* lse,
                                  void* stream) {
  return prefill_entry(cache, q, num_q_heads, gqa_group, cu_q_lens, page_table,
                       max_pages_per_seq, seq_lens, num_chunks, total_q, max_q_len,
                       softmax_scale, out, lse, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
