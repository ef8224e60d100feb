// Decode attention for callers that cannot allocate device memory.
//
// paged_decode_attention needs a caller-provided workspace for its split
// partials and per-unit records.  Some callers have no way to obtain one:
// code running where cudaMalloc is forbidden or unavailable (inside a host
// callback or a foreign runtime that owns all allocations, an embedded or
// plugin context handed only input/output pointers), or code that must not
// change the device's allocation state at all.  For them this file offers
// paged_decode_attention_noalloc, which uses a scratch buffer that lives in
// the library itself: a file-scope __device__ array of a fixed size.
//
// Consequences a caller must know:
//  * Every GPU that loads this library holds PKV_NOALLOC_SCRATCH_BYTES of
//    device memory for the array until the process exits.
//  * All calls on one device share the array.  Two calls whose executions
//    overlap on the GPU (different streams, no ordering between them) race
//    on it and produce wrong results; order them on one stream.
//  * The array keeps whatever the last call left in it.  That is harmless:
//    every value a call reads from it was written earlier by the same call,
//    so nothing needs to start at zero.
//  * The first call on a device looks up the array's device address (host
//    code cannot use the array's name as a device pointer).  Make that first
//    call before capturing any stream into a CUDA graph.
//  * Under CUDA's default lazy module loading, the array's device memory is
//    committed by that first call on each device, not when the library
//    loads.  So the first call is the one that can fail for lack of device
//    memory (it returns PKV_ERR_CUDA).  A caller whose device memory is later
//    handed over to a foreign allocator should make one call first, while
//    memory is still free, or run with CUDA_MODULE_LOADING=EAGER, which
//    commits the array when the CUDA context is created.  Later calls
//    allocate nothing.
//  * The looked-up address is cached per device for the life of the process.
//    It does not survive a reset of the device's primary context
//    (cudaDeviceReset): do not use this entry point after one.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"

namespace pkv {

// Static decode scratch: split partials + per-unit records of paged_decode_attention.
static __device__ __align__(256) uint8_t g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once
// per device, with that device current).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return PKV_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PKV_OK;
}
}  // namespace

}  // namespace pkv

using namespace pkv;

extern "C" int paged_decode_attention_noalloc(const pkv_cache* cache, const void* q,
                                              int32_t num_q_heads, int32_t gqa_group,
                                              const int32_t* page_table,
                                              int32_t max_pages_per_seq, const int32_t* seq_lens,
                                              int32_t batch, int32_t max_seq_len,
                                              float softmax_scale, void* out, float* lse,
                                              int32_t num_ctas, void* stream) {
  int st = check_cache(cache);
  if (st) return st;
  if ((st = check_group(cache, num_q_heads, gqa_group))) return st;
  if (batch < 0 || max_pages_per_seq < 1 || max_seq_len < 0 || num_ctas < 0) return PKV_ERR_SHAPE;
  if ((st = check_table_span(cache, max_pages_per_seq))) return st;
  if (batch == 0) return PKV_OK;
  // the checks paged_decode_attention makes on its own, first: sizing the
  // scratch below already queries the device
  if (!q || !page_table || !seq_lens || !out) return PKV_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u)
    return PKV_ERR_ALIGN;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PKV_ERR_SHAPE;
  if ((int64_t)max_seq_len > (int64_t)max_pages_per_seq * cache->page_size) return PKV_ERR_SHAPE;
  const size_t need = paged_decode_workspace_bytes(batch, num_q_heads, cache->num_kv_heads,
                                                   cache->head_dim, max_seq_len, num_ctas);
  if (need == 0) return PKV_ERR_CUDA;  // the arguments passed above: the device query failed
  if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch))) return st;
  return paged_decode_attention(cache, q, num_q_heads, gqa_group, page_table, max_pages_per_seq,
                                seq_lens, batch, max_seq_len, softmax_scale, out, lse, scratch,
                                (size_t)PKV_NOALLOC_SCRATCH_BYTES, num_ctas, stream);
}
