// Device helpers shared by the paged-KV kernels (sm_100a only).
//
// Thin inline-PTX wrappers for the asynchronous-copy and tensor-core
// instructions the kernels use: mbarriers with bounded waits, TMA tiled loads,
// ldmatrix and mma.sync fragments, and bf16/f16 packing.  Every spin-wait here
// gives up after a bounded number of tries and reports PKV_FLAG_TIMEOUT, so no
// kernel of this library can hang a GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/paged_kv.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libpagedkv is built for sm_100a only"
#endif

namespace pkv {

// A bounded wait gives up after this many nanoseconds (%globaltimer), far
// beyond any legitimate latency, and reports PKV_FLAG_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void flag_error(int32_t* flags, int bit) {
  if (flags) atomicOr(flags, bit);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase with the given parity to complete.  With
// suspend_ns > 0 a waiting thread may sleep up to that long per try (it is
// woken when the phase completes), so an idle warp costs no issue slots.
// Returns false (and raises PKV_FLAG_TIMEOUT) after limit_ns.  Every wait of
// every kernel in this library goes through here with the default limit;
// pkv_check_bounded_wait runs the same code with a short one.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* flags,
                                          uint32_t suspend_ns = 0,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    const bool ok =
        suspend_ns ? mbar_try_wait_sleep(bar, parity, suspend_ns) : mbar_try_wait(bar, parity);
    if (ok) return true;
    if (global_ns() - t0 > limit_ns) break;
  }
  flag_error(flags, PKV_FLAG_TIMEOUT);
  return false;
}

// ---------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 2-D tiled TMA load (no multicast) into this CTA's shared memory; completion
// is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::"
      "cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Plain bulk copy (no multicast) of `bytes` contiguous bytes into this CTA's
// shared memory; both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled TMA load (no multicast).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, int32_t z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------- ldmatrix / mma.sync
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transposing load of two 16x16 matrices of bytes: lanes 0-15 give the row
// addresses (16 bytes each) of the first, lanes 16-31 those of the second.
// Thread (gid, tid4) receives in r0 the bytes of the first matrix's rows
// 4*tid4 .. 4*tid4+3 (low byte first) in column gid, in r1 the same rows in
// column gid + 8, and in r2, r3 the same of the second matrix (lane layout
// checked on B200 with an in-bounds probe).
__device__ __forceinline__ void ldsm_x2_t_b8(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                             uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D with bf16 inputs and fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same with f16 inputs.
__device__ __forceinline__ void mma_f16(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A(16x32, row) * B(32x8, col) + D with signed 8-bit operands and exact
// s32 accumulate, rows 8-15 of A zero.  a0 / a2: a thread's four A bytes at
// columns 4*tid4 + {0..3} and + 16 of row gid; b0 / b1: its four B bytes at
// rows 4*tid4 + {0..3} and + 16 of column gid (low byte first).
__device__ __forceinline__ void mma_s8(int32_t* d, uint32_t a0, uint32_t a2, uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Same with all four A registers (rows gid + 8 in a1 / a3).
__device__ __forceinline__ void mma_s8_full(int32_t* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 matrix of 16-bit elements held one row pair per
// thread (row gid, columns 2*tid4 and 2*tid4 + 1, low half first): the
// thread receives row gid, columns 2*tid4 and 2*tid4 + 1 of the transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

// ------------------------------------------------------------------ packing
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two E4M3 codes (low byte = element 0) to an f16x2 (exact conversion).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t codes) {
  uint32_t out;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(codes));
  return out;
}

// Two INT8 codes (low byte = element 0) to an f16x2, exactly.  Flipping the
// sign bit of a two's-complement byte q gives the unsigned byte q + 128; put
// under the f16 exponent of 1024 (bits 0x64xx) it reads 1024 + q + 128, and
// subtracting 1152 leaves q (every integer up to 2048 is an f16).
__device__ __forceinline__ uint32_t s8x2_to_f16x2(uint16_t codes) {
  const uint32_t u = (uint32_t)codes ^ 0x8080u;
  uint32_t v = __byte_perm(u, 0x6464u, 0x4140);  // bytes: u0, 0x64, u1, 0x64
  const uint32_t bias = 0x64806480u;             // f16x2 {1152, 1152}
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(v) : "r"(v), "r"(bias));
  return v;
}

// Symmetric INT8 code of a quotient: round to nearest even, clamp to +-127,
// NaN stored as 0.
__device__ __forceinline__ uint32_t int8_code(float y) {
  if (y != y) return 0u;
  const int q = __float2int_rn(fminf(fmaxf(y, -127.f), 127.f));
  return static_cast<uint32_t>(q) & 0xffu;
}

// Codes of pool format kFmt for two bf16 values and their (page, head) scale
// (low byte = first value): the IEEE fp32 quotient x / scale, then E4M3 with
// round-to-nearest-even and satfinite, or the INT8 code above.  Every writer
// of one-byte pools goes through here, so all write the same bytes.
template <int kFmt>
__device__ __forceinline__ uint16_t encode8x2(__nv_bfloat162 x, float scale) {
  float2 f = __bfloat1622float2(x);
  f.x = __fdiv_rn(f.x, scale);
  f.y = __fdiv_rn(f.y, scale);
  if constexpr (kFmt == PKV_KV_INT8)
    return static_cast<uint16_t>(int8_code(f.x) | (int8_code(f.y) << 8));
  else
    return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3));
}

// Four 8-bit KV codes of format kFmt (one 32-bit word, byte 0 first) to two
// f16x2: lo = codes 0, 1 and hi = codes 2, 3 (exact for both formats).  INT8
// flips the four sign bits at once, then puts each code under the f16
// exponent of 1024 as s8x2_to_f16x2 does; E4M3 converts each 16-bit half.
template <int kFmt>
__device__ __forceinline__ void kv8x4_to_f16x2(uint32_t codes, uint32_t& lo, uint32_t& hi) {
  if constexpr (kFmt == PKV_KV_INT8) {
    const uint32_t u = codes ^ 0x80808080u;
    const uint32_t bias = 0x64806480u;  // f16x2 {1152, 1152}
    lo = __byte_perm(u, 0x6464u, 0x4140);  // bytes: u0, 0x64, u1, 0x64
    hi = __byte_perm(u, 0x6464u, 0x4342);  // bytes: u2, 0x64, u3, 0x64
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(lo), "r"(bias));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(hi), "r"(bias));
  } else {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(codes));
  }
}

// Two 8-bit KV codes of format kFmt to an f16x2 (exact for both formats).
template <int kFmt>
__device__ __forceinline__ uint32_t kv8x2_to_f16x2(uint16_t codes) {
  if constexpr (kFmt == PKV_KV_INT8)
    return s8x2_to_f16x2(codes);
  else
    return e4m3x2_to_f16x2(codes);
}

// ------------------------------------------------------------ FP4 (E2M1)
// E2M1 code of y (1 sign, 2 exponent bits with bias 1, 1 mantissa bit:
// magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), nearest with ties to the even
// code, |y| >= 6 saturating to 6, NaN as +0.  The magnitude code counts the
// midpoints between neighbours that |y| lies above; a midpoint itself goes
// to the even neighbour, hence '>' towards an even upper code's left and '>='
// where the upper neighbour is the even one.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  if (y != y) return 0u;
  const float a = fabsf(y);
  const uint32_t m = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
                     (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) +
                     (uint32_t)(a > 5.0f);
  return m | (__float_as_uint(y) >> 31 << 3);
}

// One FP4 block: 16 bf16 values (lo = elements 0-7, hi = 8-15) under the
// (page, kv head) scale s.  sb = e4m3_rne_satfinite(amax / fp32(6 s)) with
// NaN ignored in amax; d = fp32(decode(sb) * s); code_i =
// e2m1(d > 0 ? fp32(x_i / d) : 0).  Returns the 8 code bytes (element 2k in
// the low nibble of byte k) and the block-scale byte.  Every writer of FP4
// pools goes through here, so all write the same bytes.
__device__ __forceinline__ uint2 nvfp4_encode_block(const uint4& lo, const uint4& hi, float s,
                                                    uint32_t* sb_out) {
  float x[16];
  const __nv_bfloat162* p0 = reinterpret_cast<const __nv_bfloat162*>(&lo);
  const __nv_bfloat162* p1 = reinterpret_cast<const __nv_bfloat162*>(&hi);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 a = __bfloat1622float2(p0[k]);
    const float2 b = __bfloat1622float2(p1[k]);
    x[2 * k] = a.x;
    x[2 * k + 1] = a.y;
    x[8 + 2 * k] = b.x;
    x[8 + 2 * k + 1] = b.y;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));  // fmaxf drops NaN
  const float ratio = __fdiv_rn(amax, __fmul_rn(6.0f, s));
  const uint32_t sb = (uint32_t)__nv_cvt_float_to_fp8(ratio, __NV_SATFINITE, __NV_E4M3);
  __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sb, __NV_E4M3);
  const float d = __fmul_rn(__half2float(__half(hr)), s);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t c = e2m1_code(d > 0.f ? __fdiv_rn(x[i], d) : 0.f);
    w[i >> 3] |= c << (4 * (i & 7));
  }
  *sb_out = sb;
  return make_uint2(w[0], w[1]);
}

// Four bytes of E2M1 code pairs to four f16x2 (exact; the low nibble of a
// byte becomes the low half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t* out) {
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, c3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(codes));
}

// The E4M3 block-scale byte k (0-3) of `word` as an f16x2 with that value in
// both halves (exact).
__device__ __forceinline__ uint32_t e4m3_splat_f16x2(uint32_t word, uint32_t k) {
  return e4m3x2_to_f16x2((uint16_t)__byte_perm(word, 0u, k | (k << 4)));
}

// Two E4M3 bytes (k0 of word a, k1 of word b) as an f16x2 {a.k0, b.k1}.
__device__ __forceinline__ uint32_t e4m3_pair_f16x2(uint32_t a, uint32_t k0, uint32_t b,
                                                    uint32_t k1) {
  return e4m3x2_to_f16x2((uint16_t)__byte_perm(a, b, k0 | ((k1 + 4) << 4)));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// 2^x on the MUFU unit (flush-to-zero for tiny results).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Offset of byte `off` of a row-major tile after the TMA 128-byte swizzle
// (16-byte chunk index XOR row-within-8); the tile base is 1024-byte aligned.
__device__ __forceinline__ uint32_t swz128(uint32_t off) {
  return off ^ (((off >> 7) & 7u) << 4);
}

// Same for the 64-byte swizzle (512-byte aligned tile base).
__device__ __forceinline__ uint32_t swz64(uint32_t off) { return off ^ (((off >> 7) & 3u) << 4); }

// Same for the 32-byte swizzle (256-byte aligned tile base).
__device__ __forceinline__ uint32_t swz32(uint32_t off) { return off ^ (((off >> 7) & 1u) << 4); }

}  // namespace pkv
