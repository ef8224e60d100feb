// Paged KV append: the paged store of this step's new tokens.
//
// TensorRT-LLM concept page, "PagedAttention 及 KV 快取管理" and
// "編譯期圖最佳化": the K/V of a token is written to the physical page that the
// sequence's page table names for the token's logical position.
//
// One thread moves one 16-byte vector (8 bf16) of one token's K or V row:
// loads are coalesced over [token][kv head][d]; each warp writes whole
// 16-byte chunks of a contiguous page row.  bf16 pools receive the bits;
// E4M3 pools receive e4m3_rne_satfinite(x / scale) computed with an IEEE
// fp32 division and the hardware satfinite conversion; INT8 pools receive the
// nearest integer (ties to even) of the same quotient clamped to +-127, NaN
// stored as 0 (concept page, "關鍵機制", INT8 KV-cache quantisation); FP4
// pools receive E2M1 codes and E4M3 block scales per 16 values (solosoft
// post, FAQ: FP4 quantisation on Blackwell).
#include "common.cuh"
#include "kernels.h"

namespace pkv {


// Index of the sequence owning new token `tok`: the last b with cu_new[b] <= tok.
__device__ __forceinline__ int owner_of(const int32_t* cu_new, int batch, int tok) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_new + mid) <= tok)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

template <int kFmt>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  const int vecs_per_row = p.head_dim / 8;                 // 16-byte vectors per (token, head)
  const int64_t per_token = (int64_t)p.num_kv_heads * vecs_per_row;
  const int64_t total = (int64_t)p.total_new * per_token;  // vectors of K (and of V)
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < 2 * total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const bool is_v = i >= total;
    const int64_t e = is_v ? i - total : i;
    const int tok = static_cast<int>(e / per_token);
    const int rem = static_cast<int>(e - (int64_t)tok * per_token);
    const int g = rem / vecs_per_row;
    const int vec = rem - g * vecs_per_row;

    const int b = owner_of(p.cu_new, p.batch, tok);
    const int64_t pos = (int64_t)__ldg(p.seq_lens_before + b) + (tok - __ldg(p.cu_new + b));
    const int64_t j = pos / p.page_size;
    if (pos < 0 || j >= p.max_pages) {
      if (vec == 0 && g == 0 && !is_v) flag_error(p.flags, PKV_FLAG_BAD_LENGTH);
      continue;
    }
    const int32_t page = __ldg(p.page_table + (int64_t)b * p.max_pages + j);
    if (page < 0 || page >= p.num_pages) {
      if (vec == 0 && g == 0 && !is_v) flag_error(p.flags, PKV_FLAG_BAD_PAGE);
      continue;
    }
    const int slot = static_cast<int>(pos - j * p.page_size);
    const uint4 src = __ldg((is_v ? p.v_new : p.k_new) + e);
    // element index of the first of the 8 values inside the pool
    const int64_t dst_elem =
        (((int64_t)page * p.num_kv_heads + g) * p.page_size + slot) * p.head_dim + vec * 8;
    uint8_t* pool = is_v ? p.v_pool : p.k_pool;
    if constexpr (!k8(kFmt)) {
      *reinterpret_cast<uint4*>(pool + dst_elem * 2) = src;
    } else {
      const float s = __ldg((is_v ? p.v_scale : p.k_scale) + (int64_t)page * p.num_kv_heads + g);
      if (!(s > 0.f && s <= 32768.f)) {
        if (vec == 0) flag_error(p.flags, PKV_FLAG_BAD_SCALE);
      }
      const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&src);
      uint32_t w[2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint16_t two = encode8x2<kFmt>(x[k], s);
        if (k & 1)
          w[k >> 1] |= static_cast<uint32_t>(two) << 16;
        else
          w[k >> 1] = two;
      }
      *reinterpret_cast<uint2*>(pool + dst_elem) = make_uint2(w[0], w[1]);
    }
  }
}

// FP4 pools: one thread quantises one 16-element block of one token's K or
// V row (nvfp4_encode_block): 8 bytes of E2M1 codes into the row's code
// region, one E4M3 block scale into its block-scale region.
__global__ void __launch_bounds__(256) append_fp4_kernel(AppendParams p) {
  const int blocks_per_row = p.head_dim / 16;
  const int64_t per_token = (int64_t)p.num_kv_heads * blocks_per_row;
  const int64_t total = (int64_t)p.total_new * per_token;  // blocks of K (and of V)
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < 2 * total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const bool is_v = i >= total;
    const int64_t e = is_v ? i - total : i;
    const int tok = static_cast<int>(e / per_token);
    const int rem = static_cast<int>(e - (int64_t)tok * per_token);
    const int g = rem / blocks_per_row;
    const int blk = rem - g * blocks_per_row;

    const int b = owner_of(p.cu_new, p.batch, tok);
    const int64_t pos = (int64_t)__ldg(p.seq_lens_before + b) + (tok - __ldg(p.cu_new + b));
    const int64_t j = pos / p.page_size;
    if (pos < 0 || j >= p.max_pages) {
      if (blk == 0 && g == 0 && !is_v) flag_error(p.flags, PKV_FLAG_BAD_LENGTH);
      continue;
    }
    const int32_t page = __ldg(p.page_table + (int64_t)b * p.max_pages + j);
    if (page < 0 || page >= p.num_pages) {
      if (blk == 0 && g == 0 && !is_v) flag_error(p.flags, PKV_FLAG_BAD_PAGE);
      continue;
    }
    const int slot = static_cast<int>(pos - j * p.page_size);
    const float s = __ldg((is_v ? p.v_scale : p.k_scale) + (int64_t)page * p.num_kv_heads + g);
    if (!(s > 0.f && s <= 32768.f) && blk == 0) flag_error(p.flags, PKV_FLAG_BAD_SCALE);
    // source: 16 bf16 = two 16-byte vectors of the [T][Hkv][D] input
    const uint4* src = (is_v ? p.v_new : p.k_new) + e * 2;
    uint32_t sb;
    const uint2 codes = nvfp4_encode_block(__ldg(src), __ldg(src + 1), s, &sb);
    const int64_t row = ((int64_t)page * p.num_kv_heads + g) * p.page_size + slot;
    *reinterpret_cast<uint2*>((is_v ? p.v_pool : p.k_pool) + row * (p.head_dim / 2) + blk * 8) =
        codes;
    (is_v ? p.v_blocks : p.k_blocks)[row * blocks_per_row + blk] = static_cast<uint8_t>(sb);
  }
}

cudaError_t launch_append(const AppendParams& p, int fmt, int num_sms, cudaStream_t stream) {
  const int threads = 256;
  const int64_t cap = (int64_t)num_sms * 8;
  if (fmt == PKV_KV_NVFP4) {
    const int64_t units = 2LL * p.total_new * p.num_kv_heads * (p.head_dim / 16);
    if (units == 0) return cudaSuccess;
    int64_t blocks = (units + threads - 1) / threads;
    if (blocks > cap) blocks = cap;
    append_fp4_kernel<<<(unsigned)blocks, threads, 0, stream>>>(p);
    return cudaGetLastError();
  }
  const int64_t vectors = 2LL * p.total_new * p.num_kv_heads * (p.head_dim / 8);
  if (vectors == 0) return cudaSuccess;
  int64_t blocks = (vectors + threads - 1) / threads;
  if (blocks > cap) blocks = cap;
  if (fmt == PKV_KV_INT8)
    append_kernel<PKV_KV_INT8><<<(unsigned)blocks, threads, 0, stream>>>(p);
  else if (fmt == PKV_KV_FP8_E4M3)
    append_kernel<PKV_KV_FP8_E4M3><<<(unsigned)blocks, threads, 0, stream>>>(p);
  else
    append_kernel<PKV_KV_BF16><<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pkv
