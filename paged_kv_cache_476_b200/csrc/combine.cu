// Merge of attention results computed over disjoint key ranges.
//
// When the pages of one sequence are split across GPUs (or across calls),
// each part r yields the normalised output out_r and its log-sum-exp lse_r
// over its own keys.  The attention over all keys is their softmax-weighted
// combination (the split-KV reduction; the pages have no counterpart):
//   LSE = log sum_r exp(lse_r),  out = sum_r exp(lse_r - LSE) out_r.
// A part that saw no key has lse_r = -inf and weight 0; if every part is
// empty the row is 0 with lse -inf.
//
// One warp per (sequence, q head) row, lanes over head_dim; the parts are
// read once and the row written once (a few KB per sequence: launch-bound).
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"

namespace pkv {

template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ parts,
                                                      const float* __restrict__ lse_parts,
                                                      int num_parts, int rows,
                                                      __nv_bfloat16* __restrict__ out,
                                                      float* __restrict__ lse) {
  constexpr int kPer = D / 32;  // elements per lane: 2 or 4
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int r = 0; r < num_parts; ++r) m = fmaxf(m, __ldg(lse_parts + (int64_t)r * rows + row));
  float acc[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int r = 0; r < num_parts; ++r) {
      const float lr = __ldg(lse_parts + (int64_t)r * rows + row);
      const float w = expf(lr - m);  // 0 for an empty part
      wsum += w;
      const __nv_bfloat16* src = parts + ((int64_t)r * rows + row) * D + lane * kPer;
      if constexpr (kPer == 4) {
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        acc[0] += w * a.x;
        acc[1] += w * a.y;
        acc[2] += w * b.x;
        acc[3] += w * b.y;
      } else {
        const uint32_t raw = __ldg(reinterpret_cast<const unsigned int*>(src));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
        acc[0] += w * a.x;
        acc[1] += w * a.y;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = out + (int64_t)row * D + lane * kPer;
#pragma unroll
  for (int i = 0; i < kPer; i += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(acc[i] * inv, acc[i + 1] * inv);
  if (lse && lane == 0) lse[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

cudaError_t launch_combine(const void* parts, const float* lse_parts, int num_parts, int rows,
                           int head_dim, void* out, float* lse, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (rows + threads / 32 - 1) / (threads / 32);
  const auto* p = static_cast<const __nv_bfloat16*>(parts);
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (head_dim == 128)
    combine_kernel<128><<<blocks, threads, 0, stream>>>(p, lse_parts, num_parts, rows, o, lse);
  else
    combine_kernel<64><<<blocks, threads, 0, stream>>>(p, lse_parts, num_parts, rows, o, lse);
  return cudaGetLastError();
}

}  // namespace pkv
