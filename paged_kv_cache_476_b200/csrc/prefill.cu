// Causal prefill-chunk attention over a paged KV cache (sm_100a, tcgen05).
//
// What it computes (TensorRT-LLM concept page, "關鍵效能引數": context tokens
// are processed in parallel over the paged cache; "PagedAttention 及 KV 快取
// 管理": K/V pages found through the page table): for chunk c with n queries
// over L cached tokens, query i at position p = L - n + i attends to keys
// 0..p, out = softmax(scale * q K^T) V.
//
// Design (tensor-bound, B200-first):
//  * One CTA per (pair of 128-row Q tiles A and B, kv head, chunk).  The 128
//    rows of a tile pack the G q heads of the kv head for 128/G consecutive
//    query tokens (row = token * G + head), so every K/V tile staged in
//    shared memory serves the whole GQA group and both Q tiles.
//  * CTAs take their items longest-first (most KV tiles first), so the short
//    items fill the tail of the grid instead of the long ones.
//  * Warp 8 (producer) loads the two Q tiles once with a 3-D TMA map over
//    [token][head][d] and streams 128-key K/V tiles (one 128-token page or
//    two 64-token pages, page-table indirected, 128-byte swizzled) into
//    two-slot K and V rings; a K slot frees as soon as both S products have
//    read it, so the next K streams in a whole tile ahead, and the page
//    lookup of the next tile runs before the slot wait.
//  * Warp 9 (one elected thread) issues tcgen05.mma: S = Q K^T (M=128,
//    N=128, K=head_dim, both operands K-major from shared memory) into the
//    tile's TMEM S buffer, then O += P V with P (16-bit) read from TMEM over
//    S and V as an MN-major operand.  tcgen05.commit signals completion on
//    mbarriers.  The two tiles alternate, so one tile's softmax runs under
//    the other tile's products.
//  * Warps 0-3 (tile A) and 4-7 (tile B), one TMEM lane = one row per
//    thread, run the online softmax: load S from TMEM, mask the causal
//    diagonal, keep a reference max that is raised only when a row's max
//    grows by more than 2^8 (then O is rescaled in TMEM), write P to TMEM,
//    and finally normalise O.
//  * V rows past the sequence end (or of a rejected page) are zeroed in
//    shared memory before their PV product: 0 * NaN would poison O.
//  * E4M3 and INT8 pools: two converter warps turn each landed tile of
//    one-byte codes into a 16-bit tile (exact) laid out as TMA lays out bf16
//    tiles: K as bf16 (Q's type), V as f16.  The per-(page, head) K scales multiply the scores of their
//    64-key block; the V scales ride on P, kept in f16 (11-bit mantissa) so
//    that PV is an f16 x f16 product.
//  * Every wait is bounded; TMEM is freed on every exit path.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pkv {

namespace pf {

constexpr int kRows = 128;     // M of a Q tile; a CTA holds two Q tiles, A and B
constexpr int kKeys = 128;     // N of the S tile (keys per KV tile)
constexpr int kStages = 2;     // K/V ring depth
// warps 0-3 softmax of Q tile A, 4-7 softmax of Q tile B (one TMEM lane =
// one row per thread), 8 producer, 9 MMA, 10-11 E4M3 converters (E4M3 only)
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp0 = 10;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S of tile A and B (P is written over S as 16-bit pairs), O
// of tile A and B.
__device__ __forceinline__ uint32_t col_s(int x) { return x ? 128u : 0u; }
__device__ __forceinline__ uint32_t col_o(int x) { return x ? 384u : 256u; }

struct Params {
  const float* k_scale;  // [pages][Hkv] (quantised pools)
  const float* v_scale;
  const uint8_t* k_blocks;  // FP4 pools: the block-scale regions (after the codes)
  const uint8_t* v_blocks;
  const int32_t* cu_q;
  const int32_t* page_table;
  const int32_t* seq_lens;
  __nv_bfloat16* out;  // [Tq][Hq][D]
  float* lse;          // [Tq][Hq] or null
  int32_t* flags;
  int32_t num_chunks;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t group;
  int32_t max_pages;
  int32_t num_pages;
  int32_t page_size;
  int32_t pair_slots;  // pairs of Q tiles per chunk the grid provides
  int32_t lpt;         // 1: longest-first item order, 0: index order
  float scale_log2;
};

// --------------------------------------------------------- tcgen05 helpers
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Store 16 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// max(a, b, c) in one instruction (three-input form of sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Two fp32 lanes at once (sm_100 packed FMA / add / mul): each lane rounds
// exactly as its scalar instruction would.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}

// O row (this thread's TMEM lane, D fp32 columns from taddr) *= alpha.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t taddr, float alpha) {
#pragma unroll
  for (int c = 0; c < D; c += 32) {
    float o[32];
    tmem_ld32(taddr + c, o);
    tmem_wait_ld();
    uint32_t u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * alpha);
    tmem_st16(taddr + c, u);
    tmem_st16(taddr + c + 16, u + 16);
  }
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading
// and stride byte offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16 with f32 accumulation: A and B both
// bf16 (or both f16), M x N, B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc_f16kind(int M, int N, int b_mn_major, bool bf16) {
  return (1u << 4)                           // D format f32
         | ((bf16 ? 1u : 0u) << 7)           // A: 1 bf16, 0 f16
         | ((bf16 ? 1u : 0u) << 10)          // B: same type as A
         | ((uint32_t)b_mn_major << 16)      // B major: 0 K, 1 MN
         | ((uint32_t)(N >> 3) << 17)        // N / 8
         | ((uint32_t)(M >> 4) << 24);       // M / 16
}

template <int D, int kFmt>
struct Smem {
  static constexpr int kHalves = D / 64;            // 128-byte column boxes per bf16 row
  static constexpr int kQB = kRows * D * 2;         // one Q tile
  static constexpr int kTileB = kKeys * D * 2;      // bf16 K (or V) tile
  static constexpr int kHalfB = kKeys * 128;        // one 64-column half of a bf16 tile
  // a quantised K (or V) tile as it lands: the codes of its rows, then (FP4)
  // their block scales
  static constexpr int kCodeRowB = row_code_bytes(kFmt, D);
  static constexpr int kScaleRowB = row_scale_bytes(kFmt, D);
  static constexpr int kCodesB = kKeys * kCodeRowB;
  static constexpr int kTileQB = kCodesB + kKeys * kScaleRowB;
  static constexpr int kStageB = quant(kFmt) ? 2 * kTileQB : 2 * kTileB;
  static constexpr int kConvB = quant(kFmt) ? 2 * kTileB : 0;  // converted K, then V
  static constexpr int kBytes = 2 * kQB + kStages * kStageB + kConvB;
  static constexpr int kThreads = quant(kFmt) ? 384 : 320;  // + two converter warps
};

// Per-KV-tile facts the producer passes on: rejected 64-key blocks and the
// E4M3 scales of the (up to two) pages of the tile.
struct TileFacts {
  int32_t bad;
  float ks[2], vs[2];
};
constexpr int kFactsRing = 4;

// Shared-memory byte address of 16-byte chunk c (0..D/8-1) of row r of a bf16
// tile laid out as TMA writes it: 64-column halves kHalfB apart, 128-byte
// rows, 128-byte swizzle.
template <int D>
__device__ __forceinline__ uint32_t bf16_chunk(uint32_t base, int r, int c) {
  return base + (c >> 3) * (kKeys * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// Same for a tile of codes as TMA writes it: rows of kRowB bytes with the
// swizzle of that width (128, 64 or 32 bytes).
template <int kRowB>
__device__ __forceinline__ uint32_t code_chunk(uint32_t base, int r, int c) {
  if constexpr (kRowB == 128)
    return base + r * 128 + ((c ^ (r & 7)) << 4);
  else if constexpr (kRowB == 64)
    return base + r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
  else
    return base + r * 32 + ((c ^ ((r >> 2) & 1)) << 4);
}

// E4M3 tile -> bf16 or f16 tile (both exact: every E4M3 value is an f16 and a
// bf16), rows in `zero_mask` (bit per 64-row block) or at/after `zero_from`
// written as zeros.  64 threads share the work.
template <int D, int kFmt, bool kToF16>
__device__ __forceinline__ void convert_tile(uint32_t src, uint32_t dst, int t, int zero_from,
                                             int zero_mask) {
  constexpr int kChunks = kKeys * D / 16;  // 16-byte E4M3 chunks
#pragma unroll 4
  for (int ci = t; ci < kChunks; ci += 64) {
    const int r = ci / (D / 16);
    const int c = ci - r * (D / 16);
    uint32_t o[8];
    if (r >= zero_from || ((zero_mask >> (r >> 6)) & 1)) {
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = 0u;
    } else {
      uint32_t w[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                   : "r"(code_chunk<D>(src, r, c)));
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t h01 = kv8x2_to_f16x2<kFmt>(w[k] & 0xffff);
        const uint32_t h23 = kv8x2_to_f16x2<kFmt>(w[k] >> 16);
        if constexpr (kToF16) {
          o[2 * k] = h01;
          o[2 * k + 1] = h23;
        } else {
          const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
          const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
          o[2 * k] = pack_bf16(f01.x, f01.y);
          o[2 * k + 1] = pack_bf16(f23.x, f23.y);
        }
      }
    }
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(bf16_chunk<D>(dst, r, 2 * c)),
                 "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                 : "memory");
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                     bf16_chunk<D>(dst, r, 2 * c + 1)),
                 "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                 : "memory");
  }
}

// FP4 tile (codes, then one E4M3 block scale per 16 values of a row) ->
// bf16 or f16 tile, values e2m1(code) * decode(sb): exact in both, since the
// product has at most 6 significant bits and lies in [2^-10, 2688].  Rows
// in `zero_mask` or at/after `zero_from` are written as zeros.  64 threads.
template <int D, bool kToF16>
__device__ __forceinline__ void convert_fp4_tile(uint32_t src, uint32_t dst, int t, int zero_from,
                                                 int zero_mask) {
  constexpr int kRowB = D / 2;            // code bytes of a row
  constexpr int kChunks = kKeys * D / 32;  // 16-byte chunks of codes (32 values, 2 blocks)
  const uint32_t scales = src + kKeys * kRowB;
#pragma unroll 2
  for (int ci = t; ci < kChunks; ci += 64) {
    const int r = ci / (D / 32);
    const int c = ci - r * (D / 32);
    uint32_t o[16];
    if (r >= zero_from || ((zero_mask >> (r >> 6)) & 1)) {
#pragma unroll
      for (int k = 0; k < 16; ++k) o[k] = 0u;
    } else {
      uint32_t w[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                   : "r"(code_chunk<kRowB>(src, r, c)));
      uint32_t sb2;
      asm volatile("ld.shared.u16 %0, [%1];" : "=r"(sb2) : "r"(scales + r * (D / 16) + 2 * c));
      const uint32_t s0 = e4m3_splat_f16x2(sb2, 0), s1 = e4m3_splat_f16x2(sb2, 1);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        e2m1x8_to_f16x2(w[k], o + 4 * k);
#pragma unroll
        for (int i = 0; i < 4; ++i) o[4 * k + i] = hmul2_u32(o[4 * k + i], k < 2 ? s0 : s1);
      }
      if constexpr (!kToF16) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&o[k]));
          o[k] = pack_bf16(f.x, f.y);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(bf16_chunk<D>(dst, r, 4 * c + q)),
                   "r"(o[4 * q]), "r"(o[4 * q + 1]), "r"(o[4 * q + 2]), "r"(o[4 * q + 3])
                   : "memory");
  }
}

// ------------------------------------------------- longest-first CTA order
// A work item is (chunk, pair of Q tiles); its cost is the number of KV tiles
// its later tile visits, ceil((ctx + e) / 128) with ctx = L - n and e the end
// of the pair inside the chunk, min(2 TQ (pair + 1), n): nondecreasing in the
// pair index.  The hardware dispatches CTAs in index order onto whichever SM
// frees first, so handing out items by descending cost is the greedy
// longest-processing-time schedule.  Each CTA derives its item from its rank
// with a warp-wide count: no plan buffer, no host knowledge of lengths.
constexpr int kLptChunksPerLane = 4;
constexpr int kLptMaxChunks = 32 * kLptChunksPerLane;  // more chunks: index order

struct ChunkCost {
  int32_t ctx, n, pairs;  // pairs: items of the chunk that exist in the grid
};

// Items of chunk `cc` whose cost is below k.  Straight-line: the warp runs
// it for every chunk slot at every step of the search, and branches there
// split the lanes.
__device__ __forceinline__ int32_t pairs_below(const ChunkCost& cc, int32_t k, int32_t pair_tokens) {
  const int64_t lim = (int64_t)kKeys * (k - 1) - cc.ctx;  // cost < k  <=>  ctx + e <= lim
  // clamped to [0, n] (n < 2^31), so that a 32-bit division serves
  const uint32_t v = (uint32_t)max(min(lim, (int64_t)cc.n), (int64_t)0);
  const int32_t q = min((int32_t)(v / (uint32_t)pair_tokens), cc.pairs);
  return lim >= cc.n ? cc.pairs : q;
}

// Sum over the warp's chunks of the items with cost >= k.
__device__ __forceinline__ uint32_t items_at_least(const ChunkCost* cc, int32_t k,
                                                   int32_t pair_tokens) {
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < kLptChunksPerLane; ++i)
    s += (uint32_t)(cc[i].pairs - pairs_below(cc[i], k, pair_tokens));
  return __reduce_add_sync(0xffffffffu, s);
}

// Warp 0: the item of rank `rank` in descending-cost order (ties by chunk
// index, then pair index).  Returns false when the rank is past the last item.
__device__ bool lpt_item(const Params& p, uint32_t rank, int32_t pair_tokens, int32_t* chunk_out,
                         int32_t* pair_out) {
  const int lane = threadIdx.x & 31;
  ChunkCost cc[kLptChunksPerLane];
  int32_t kmax = 0;
#pragma unroll
  for (int i = 0; i < kLptChunksPerLane; ++i) {
    const int c = lane * kLptChunksPerLane + i;
    cc[i].ctx = cc[i].n = cc[i].pairs = 0;
    if (c < p.num_chunks) {
      const int32_t n = max(__ldg(p.cu_q + c + 1) - __ldg(p.cu_q + c), 0);
      const int32_t L = __ldg(p.seq_lens + c);
      cc[i].n = n;
      cc[i].ctx = (int32_t)max((int64_t)L - n, (int64_t)0);
      cc[i].pairs = min((int32_t)(((uint32_t)n + pair_tokens - 1) / (uint32_t)pair_tokens), p.pair_slots);
      kmax = max(kmax, (int32_t)(((int64_t)cc[i].ctx + n + kKeys - 1) / kKeys));
    }
  }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (items_at_least(cc, 1, pair_tokens) <= rank) return false;
  // largest k with more than `rank` items of cost >= k
  int32_t lo = 1, hi = kmax + 1;
  while (hi - lo > 1) {
    const int32_t mid = lo + (hi - lo) / 2;
    if (items_at_least(cc, mid, pair_tokens) > rank)
      lo = mid;
    else
      hi = mid;
  }
  uint32_t o = rank - items_at_least(cc, lo + 1, pair_tokens);  // offset among cost == lo
  int32_t below[kLptChunksPerLane];
  uint32_t eq[kLptChunksPerLane], mine = 0;
#pragma unroll
  for (int i = 0; i < kLptChunksPerLane; ++i) {
    below[i] = pairs_below(cc[i], lo, pair_tokens);
    eq[i] = (uint32_t)(pairs_below(cc[i], lo + 1, pair_tokens) - below[i]);
    mine += eq[i];
  }
  uint32_t incl = mine;  // inclusive scan over lanes (chunks are lane-major)
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  const uint32_t excl = incl - mine;
  const uint32_t hit = __ballot_sync(0xffffffffu, excl <= o && o < incl);
  const int owner = __ffs(hit) - 1;  // exists: the counts above add up past o
  int32_t c_sel = 0, pr_sel = 0;
  if (lane == owner) {
    o -= excl;
#pragma unroll
    for (int i = 0; i < kLptChunksPerLane; ++i) {
      if (o < eq[i]) {
        c_sel = lane * kLptChunksPerLane + i;
        pr_sel = below[i] + (int32_t)o;
        break;
      }
      o -= eq[i];
    }
  }
  *chunk_out = __shfl_sync(0xffffffffu, c_sel, owner);
  *pair_out = __shfl_sync(0xffffffffu, pr_sel, owner);
  return true;
}

template <int D, int kFmt>
__global__ void __launch_bounds__(Smem<D, kFmt>::kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using Sm = Smem<D, kFmt>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = smem;                               // Q tile A, then Q tile B
  uint8_t* skv = smem + 2 * Sm::kQB;                // stage s: K at s*kStageB, V after it
  uint8_t* sconv = skv + kStages * Sm::kStageB;     // E4M3 only: 16-bit K, then V
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sm::kBytes);
  uint64_t* q_full = bars + 0;
  // K and V have rings of their own: K(j) is free once both S products of
  // tile j ran, long before V(j) is, so K(j + 2) streams in early.
  uint64_t* k_full = bars + 1;                // [kStages] TMA landed
  uint64_t* k_empty = k_full + kStages;       // [kStages] slot may be refilled
  uint64_t* v_full = k_empty + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_full = v_empty + kStages;       // [2] S of tile A / B computed
  uint64_t* p_full = s_full + 2;              // [2] P of tile A / B written
  uint64_t* o_bar = p_full + 2;               // [2] PV of tile A / B done
  uint64_t* done_bar = o_bar + 2;
  uint64_t* kc_full = done_bar + 1;           // E4M3: converted K ready / free
  uint64_t* kc_free = kc_full + 1;
  uint64_t* vc_full = kc_free + 1;            // E4M3: converted V ready / free
  uint64_t* vc_free = vc_full + 1;
  uint64_t* facts_full = vc_free + 1;         // [kFactsRing] producer -> softmax
  TileFacts* facts = reinterpret_cast<TileFacts*>(facts_full + kFactsRing);
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(facts + kFactsRing);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.group;
  const int TQ = kRows / G;  // query tokens per Q tile
  int32_t* sched = reinterpret_cast<int32_t*>(tmem_base_smem + 1);  // chunk, pair, head

  // Item choice (warp 0), barrier set-up (warp 1) and TMEM allocation (MMA
  // warp) overlap; one barrier publishes all three.
  if (warp == 0) {
    const uint32_t lin = blockIdx.x;
    int32_t c = -1, pr = 0, hd = 0;
    if (p.lpt) {
      hd = (int32_t)(lin % (uint32_t)p.num_kv_heads);
      if (!lpt_item(p, lin / (uint32_t)p.num_kv_heads, 2 * TQ, &c, &pr)) c = -1;
    } else {
      pr = (int32_t)(lin % (uint32_t)p.pair_slots);
      hd = (int32_t)((lin / (uint32_t)p.pair_slots) % (uint32_t)p.num_kv_heads);
      c = (int32_t)(lin / ((uint32_t)p.pair_slots * (uint32_t)p.num_kv_heads));
    }
    if (lane == 0) {
      sched[0] = c;
      sched[1] = pr;
      sched[2] = hd;
    }
  }
  if (warp == 1 && lane == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], quant(kFmt) ? 2 : 1);  // quantised: released by the two converter warps
      mbar_init(&v_empty[s], quant(kFmt) ? 2 : 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 4);
      mbar_init(&o_bar[x], 1);
    }
    mbar_init(done_bar, 1);
    mbar_init(kc_full, 2);
    mbar_init(kc_free, 1);
    mbar_init(vc_full, 2);
    mbar_init(vc_free, 1);
    for (int s = 0; s < kFactsRing; ++s) mbar_init(&facts_full[s], 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_base_smem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;
  const int chunk = sched[0];
  const int g = sched[2];
  const int qa0 = sched[1] * 2 * TQ;  // first token of tile A; tile B follows

  // Decide, uniformly across the CTA, whether the item has work.
  bool run = chunk >= 0 && chunk < p.num_chunks;
  int32_t q_begin = 0, n = 0, L = 0;
  if (run) {
    q_begin = __ldg(p.cu_q + chunk);
    n = __ldg(p.cu_q + chunk + 1) - q_begin;
    L = __ldg(p.seq_lens + chunk);
    run = n > 0 && qa0 < n;
  }
  const int32_t cap = p.max_pages * p.page_size;
  if (run && (L > cap || n > L)) {
    if (threadIdx.x == 0) flag_error(p.flags, PKV_FLAG_BAD_LENGTH);
    if (n > cap || L < n) run = false;  // nothing meaningful to compute
    L = min(L, cap);
  }
  if (!run) {
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  const int q0[2] = {qa0, qa0 + TQ};
  const bool hasB = q0[1] < n;
  int nkv[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int32_t pmax = L - n + min(q0[x] + TQ, n) - 1;  // largest query position
    nkv[x] = (x == 0 || hasB) ? (pmax + kKeys) / kKeys : 0;
  }
  const int n_kv = max(nkv[0], nkv[1]);  // KV tiles the CTA visits

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      mbar_arrive_expect_tx(q_full, (uint32_t)(hasB ? 2 : 1) * Sm::kQB);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (x == 1 && !hasB) break;
#pragma unroll
        for (int h = 0; h < Sm::kHalves; ++h)
          tma_load_3d(sq + x * Sm::kQB + h * (kRows * 128), &tmap_q, h * 64, g * G,
                      q_begin + q0[x], q_full);
      }
    }
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      // Page lookup of tile j: page ids, E4M3 scales, rejected 64-key blocks.
      struct Lookup {
        TileFacts tf;
        int32_t ys[2];  // first pool row of each 64-key block
        int live;       // bit per 64-key block with data to load
      };
      auto lookup = [&](int j) -> Lookup {
        Lookup lk;
        lk.tf.bad = 0;
        lk.live = 0;
        for (int sb = 0; sb < 2; ++sb) {
          lk.tf.ks[sb] = lk.tf.vs[sb] = 1.f;
          lk.ys[sb] = 0;
          const int32_t key0 = j * kKeys + sb * 64;
          if (key0 >= L) continue;
          const int32_t pj = key0 / p.page_size;
          const int32_t pid = __ldg(p.page_table + (int64_t)chunk * p.max_pages + pj);
          if (pid < 0 || pid >= p.num_pages) {
            flag_error(p.flags, PKV_FLAG_BAD_PAGE);
            lk.tf.bad |= 1 << sb;
            continue;
          }
          if constexpr (quant(kFmt)) {
            const float ks = __ldg(p.k_scale + (int64_t)pid * p.num_kv_heads + g);
            const float vs = __ldg(p.v_scale + (int64_t)pid * p.num_kv_heads + g);
            if (!(ks > 0.f && ks <= 32768.f && vs > 0.f && vs <= 32768.f)) {
              flag_error(p.flags, PKV_FLAG_BAD_SCALE);
              lk.tf.bad |= 1 << sb;
              continue;
            }
            lk.tf.ks[sb] = ks;
            lk.tf.vs[sb] = vs;
          }
          lk.ys[sb] = (int32_t)(((int64_t)pid * p.num_kv_heads + g) * p.page_size +
                                key0 % p.page_size);
          lk.live |= 1 << sb;
        }
        return lk;
      };
      // bytes of one operand (K or V) per live 64-key block
      constexpr uint32_t kBlockBytes =
          quant(kFmt) ? 64u * (Sm::kCodeRowB + Sm::kScaleRowB) : Sm::kHalves * 64u * 128u;
      // load one operand of a tile into its slot
      auto load = [&](const CUtensorMap* map, const uint8_t* blocks, uint8_t* dst, uint64_t* bar,
                      const Lookup& lk) {
        mbar_arrive_expect_tx(bar, (uint32_t)__popc(lk.live) * kBlockBytes);
        for (int sb = 0; sb < 2; ++sb) {
          if (!((lk.live >> sb) & 1)) continue;
          if constexpr (quant(kFmt)) {
            tma_load_2d(dst + sb * 64 * Sm::kCodeRowB, map, 0, lk.ys[sb], bar, pol);
            if constexpr (fp4(kFmt))  // the block scales of the same 64 rows
              bulk_load(dst + Sm::kCodesB + sb * 64 * Sm::kScaleRowB,
                        blocks + (int64_t)lk.ys[sb] * Sm::kScaleRowB, 64u * Sm::kScaleRowB, bar);
          } else {
#pragma unroll
            for (int h = 0; h < Sm::kHalves; ++h)
              tma_load_2d(dst + h * Sm::kHalfB + sb * 64 * 128, map, h * 64, lk.ys[sb], bar,
                          pol);
          }
        }
      };
      Lookup cur = lookup(0);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % kStages;
        const uint32_t ph = (uint32_t)((j / kStages - 1) & 1);
        uint8_t* kd = skv + st * Sm::kStageB;
        uint8_t* vd = kd + Sm::kStageB / 2;
        // K(j) replaces K(j - 2), whose S products are done: every reader of
        // the facts of tile j - 4 has finished too.
        if (j >= kStages && !mbar_wait(&k_empty[st], ph, p.flags)) break;
        facts[j % kFactsRing] = cur.tf;
        mbar_arrive(&facts_full[j % kFactsRing]);
        load(&tmap_k, p.k_blocks, kd, &k_full[st], cur);
        if (j >= kStages && !mbar_wait(&v_empty[st], ph, p.flags)) break;
        load(&tmap_v, p.v_blocks, vd, &v_full[st], cur);
        if (j + 1 < n_kv) cur = lookup(j + 1);  // ahead of the next slot wait
      }
    }
  } else if (quant(kFmt) && warp >= kConvWarp0) {
    // ------------------------------------------------- E4M3 -> 16-bit converters
    const int t = threadIdx.x - kConvWarp0 * 32;  // 0..63
    const uint32_t kc = smem_u32(sconv), vc = kc + Sm::kTileB;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j % kStages;
      const uint32_t par = (uint32_t)((j / kStages) & 1);
      if (!mbar_wait(&k_full[st], par, p.flags)) break;
      const uint32_t k_codes = smem_u32(skv + st * Sm::kStageB);
      const uint32_t v_codes = k_codes + Sm::kStageB / 2;
      const int bad = facts[j % kFactsRing].bad;
      const int32_t key0 = j * kKeys;
      const int zero_from = key0 + kKeys > L ? max(0, L - key0) : kKeys;
      // K (rows that must not count are masked in the scores; keep them finite)
      if (j >= 1 && !mbar_wait(kc_free, (uint32_t)((j - 1) & 1), p.flags)) break;
      if constexpr (fp4(kFmt))
        convert_fp4_tile<D, false>(k_codes, kc, t, zero_from, bad);  // bf16, like Q
      else
        convert_tile<D, kFmt, false>(k_codes, kc, t, zero_from, bad);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(kc_full);
        mbar_arrive(&k_empty[st]);  // the E4M3 K slot may be refilled
      }
      if (!mbar_wait(&v_full[st], par, p.flags)) break;
      // V (rows that must not count are zeros: 0 * NaN would poison O)
      if (j >= 1 && !mbar_wait(vc_free, (uint32_t)((j - 1) & 1), p.flags)) break;
      if constexpr (fp4(kFmt))
        convert_fp4_tile<D, true>(v_codes, vc, t, zero_from, bad);  // f16, like P
      else
        convert_tile<D, kFmt, true>(v_codes, vc, t, zero_from, bad);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(vc_full);
        mbar_arrive(&v_empty[st]);  // the E4M3 V slot may be refilled
      }
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    // Issue order per KV tile j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the
    // tensor core always has the other tile's work while a softmax runs.
    const uint32_t id_s = idesc_f16kind(kRows, kKeys, 0, true);
    // E4M3: P (scaled by the V scales) and V are f16 for the PV product
    const uint32_t id_o = idesc_f16kind(kRows, D, 1, !quant(kFmt));
    const uint32_t q_addr = smem_u32(sq);
    bool ok = mbar_wait(q_full, 0, p.flags);
    auto k_ready = [&](int j, uint32_t* addr) -> bool {
      if constexpr (quant(kFmt)) {
        *addr = smem_u32(sconv);
        return mbar_wait(kc_full, (uint32_t)(j & 1), p.flags);
      } else {
        *addr = smem_u32(skv + (j % kStages) * Sm::kStageB);
        return mbar_wait(&k_full[j % kStages], (uint32_t)((j / kStages) & 1), p.flags);
      }
    };
    auto issue_s = [&](int x, uint32_t k_addr) {
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // A = Q, B = K, both K-major: 16-element K steps advance 32 B inside
          // a 128-byte swizzled row; the second 64 columns live kHalfB away.
          const int h = kk >> 2, w = kk & 3;
          const uint64_t ad = sdesc(q_addr + x * Sm::kQB + h * (kRows * 128) + w * 32, 16, 1024);
          const uint64_t bd = sdesc(k_addr + h * Sm::kHalfB + w * 32, 16, 1024);
          mma_ss(tmem + col_s(x), ad, bd, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[x]);
      }
      __syncwarp();
    };
    // V of tile j, made safe for the PV product (rows past the end or of a
    // rejected page zeroed); returns false on a timeout
    auto v_ready = [&](int j, uint32_t* addr) -> bool {
      if constexpr (quant(kFmt)) {
        *addr = smem_u32(sconv) + Sm::kTileB;
        return mbar_wait(vc_full, (uint32_t)(j & 1), p.flags);
      } else {
        const int st = j % kStages;
        if (!mbar_wait(&v_full[st], (uint32_t)((j / kStages) & 1), p.flags)) return false;
        const int32_t key0 = j * kKeys;
        const int bad = facts[j % kFactsRing].bad;
        int zlo = kKeys;
        if (key0 + kKeys > L) zlo = max(0, L - key0);
        uint8_t* vd = skv + st * Sm::kStageB + Sm::kTileB;
        if (zlo < kKeys || bad) {
          for (int idx = lane; idx < kKeys * Sm::kHalves * 8; idx += 32) {
            const int row = idx / (Sm::kHalves * 8);
            const int rem = idx - row * (Sm::kHalves * 8);
            const int h = rem >> 3, c = rem & 7;
            const bool z = row >= zlo || ((bad >> (row >> 6)) & 1);
            if (z)
              *reinterpret_cast<uint4*>(vd + h * Sm::kHalfB + row * 128 + c * 16) =
                  make_uint4(0, 0, 0, 0);
          }
          fence_async_smem();
          __syncwarp();
        }
        *addr = smem_u32(vd);
        return true;
      }
    };
    auto issue_pv = [&](int x, int j, uint32_t v_addr) -> bool {
      if (!mbar_wait(&p_full[x], (uint32_t)(j & 1), p.flags)) return false;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          // B = V [keys x d], MN-major: 8-key groups 1024 B apart (SBO), the
          // 64-column halves kHalfB apart (LBO).  A = P, 16-bit pairs in TMEM.
          const uint64_t bd = sdesc(v_addr + kk * 2048, Sm::kHalfB, 1024);
          mma_ts(tmem + col_o(x), tmem + col_s(x) + kk * 8, bd, id_o,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&o_bar[x]);
      }
      __syncwarp();
      return true;
    };
    uint32_t k_addr = 0;
    if (ok) ok = k_ready(0, &k_addr);
    if (ok) {
      issue_s(0, k_addr);
      if (hasB) issue_s(1, k_addr);
      if (lane == 0) tc_commit(quant(kFmt) ? kc_free : &k_empty[0]);  // K_0 is read by both S products
      __syncwarp();
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      uint32_t v_addr;
      if (!(ok = v_ready(j, &v_addr))) break;
      if (j < nkv[0] && !(ok = issue_pv(0, j, v_addr))) break;
      const bool next = j + 1 < n_kv;
      if (next && !(ok = k_ready(j + 1, &k_addr))) break;
      if (j + 1 < nkv[0]) issue_s(0, k_addr);
      if (j < nkv[1] && !(ok = issue_pv(1, j, v_addr))) break;
      // V_j is consumed once both PV products have run, K_{j+1} once both
      // S products have
      if (lane == 0) tc_commit(quant(kFmt) ? vc_free : &v_empty[j % kStages]);
      __syncwarp();
      if (j + 1 < nkv[1]) issue_s(1, k_addr);
      if (next && lane == 0) tc_commit(quant(kFmt) ? kc_free : &k_empty[(j + 1) % kStages]);
      __syncwarp();
    }
    // every MMA this thread issued must finish before TMEM is released
    if (lane == 0) tc_commit(done_bar);
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------- softmax
    const int x = warp >> 2;        // Q tile: 0 = A, 1 = B
    const int wq = warp & 3;        // TMEM lane quadrant of this warp
    if (x == 0 || hasB) {
      const int r = wq * 32 + lane;  // row of the tile = TMEM lane
      const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
      const uint32_t colS = col_s(x), colO = col_o(x);
      const int nkx = x ? nkv[1] : nkv[0];
      const int q0x = x ? q0[1] : q0[0];
      const int t_local = q0x + r / G;
      const bool row_ok = t_local < n;
      const int32_t p_min = L - n + q0x;
      const int32_t pos = row_ok ? L - n + t_local : L - n + min(q0x + TQ, n) - 1;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkx; ++j) {
        if (!mbar_wait(&s_full[x], (uint32_t)(j & 1), p.flags)) { ok = false; break; }
        if (!mbar_wait(&facts_full[j % kFactsRing], (uint32_t)((j / kFactsRing) & 1), p.flags)) {
          ok = false;
          break;
        }
        const TileFacts tf = facts[j % kFactsRing];
        tc_fence_after();
        // mask: causal diagonal (which also covers keys past the end) and
        // blocks of a rejected page; E4M3 K scales per 64-key block
        const int32_t key0 = j * kKeys;
        const bool diag = key0 + kKeys - 1 > p_min;
        const float mul0 = quant(kFmt) ? p.scale_log2 * tf.ks[0] : p.scale_log2;
        const float mul1 = quant(kFmt) ? p.scale_log2 * tf.ks[1] : p.scale_log2;
        auto scaled = [&](float v, int c) -> float {
          const bool keep = (!diag || key0 + c <= pos) && !((tf.bad >> (c >> 6)) & 1);
          return keep ? v * (c < 64 ? mul0 : mul1) : -INFINITY;
        };
        // Tiles off the diagonal without a rejected page (nearly all) take a
        // lean path: max of the raw scores, then one FMA + exp2 per element.
        // (max(s) * mul = max(s * mul) needs mul > 0; other scales go the
        // general way.)
        const bool plain = !diag && tf.bad == 0 && mul0 > 0.f && mul1 > 0.f;
        // Raise the reference max to the tile max mt when needed: lazily (p
        // <= 2^8) for bf16; for E4M3 at every increase, so that p * v_scale
        // <= 2^15 fits the f16 P.  Returns the max to subtract (0 while a row
        // has seen no key, so that its p are 0).  O is rescaled by alpha
        // after P is written (the registers of S are free by then): S(j) done
        // implies every earlier MMA is done, PV(j-1) included, and PV(j)
        // waits for this tile's P.
        float alpha = 1.f;
        auto set_max = [&](float mt) -> float {
          const bool need = mt > m_ref + (quant(kFmt) ? 0.f : 8.f);  // true on the first visible tile
          const float m_new = need ? mt : m_ref;
          if (j >= 1 && need) alpha = fast_exp2(m_ref - m_new);
          m_ref = m_new;
          return m_ref == -INFINITY ? 0.f : m_ref;
        };
        float rs = 0.f;
        {
          // Two 64-column passes: the row max, then P.
          float mt = -INFINITY;
#pragma unroll
          for (int cb = 0; cb < kKeys; cb += 64) {
            float sv[64];
            tmem_ld32(tmem + lane_base + colS + cb, sv);
            tmem_ld32(tmem + lane_base + colS + cb + 32, sv + 32);
            tmem_wait_ld();
            if (plain) {
              float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
              for (int i = 0; i < 64; i += 4) {
                m0 = fmax3(m0, sv[i], sv[i + 1]);
                m1 = fmax3(m1, sv[i + 2], sv[i + 3]);
              }
              mt = fmaxf(mt, fmaxf(m0, m1) * (cb < 64 ? mul0 : mul1));
            } else {
#pragma unroll
              for (int i = 0; i < 64; ++i) mt = fmaxf(mt, scaled(sv[i], cb + i));
            }
          }
          const float m_use = set_max(mt);
#pragma unroll
          for (int cb = 0; cb < kKeys; cb += 64) {
            float sv[64];
            tmem_ld32(tmem + lane_base + colS + cb, sv);
            tmem_ld32(tmem + lane_base + colS + cb + 32, sv + 32);
            tmem_wait_ld();
            const float mul = cb < 64 ? mul0 : mul1;
            // quantised pools: the V scales ride on P
            const float vsc = quant(kFmt) ? (cb < 64 ? tf.vs[0] : tf.vs[1]) : 1.f;
            uint32_t pk[32];
            // (two loops rather than a branch per element, which the compiler
            // would turn into both paths under predicates)
            if (plain) {
              float2 racc = make_float2(0.f, 0.f);
              const float2 mul_2 = make_float2(mul, mul), neg_2 = make_float2(-m_use, -m_use);
              const float2 vsc_2 = make_float2(vsc, vsc);
#pragma unroll
              for (int i = 0; i < 64; i += 2) {
                const float2 t = fma2(make_float2(sv[i], sv[i + 1]), mul_2, neg_2);
                const float2 pp = make_float2(fast_exp2(t.x), fast_exp2(t.y));
                racc = add2(racc, pp);
                if constexpr (quant(kFmt)) {
                  const float2 ps = mul2(pp, vsc_2);
                  pk[i / 2] = pack_f16(ps.x, ps.y);
                } else {
                  pk[i / 2] = pack_bf16(pp.x, pp.y);
                }
              }
              rs += racc.x + racc.y;
            } else {
#pragma unroll
              for (int i = 0; i < 64; i += 2) {
                const float p0 = fast_exp2(scaled(sv[i], cb + i) - m_use);
                const float p1 = fast_exp2(scaled(sv[i + 1], cb + i + 1) - m_use);
                rs += p0 + p1;
                pk[i / 2] = quant(kFmt) ? pack_f16(p0 * vsc, p1 * vsc) : pack_bf16(p0, p1);
              }
            }
            // P column c/2 lies in an S column already read
            tmem_st16(tmem + lane_base + colS + cb / 2, pk);
            tmem_st16(tmem + lane_base + colS + cb / 2 + 16, pk + 16);
          }
        }
        if (__any_sync(0xffffffffu, alpha != 1.f)) rescale_o<D>(tmem + lane_base + colO, alpha);
        l = l * alpha + rs;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
      }
      // ------------------------------------------------------ epilogue
      if (ok && nkx > 0 &&
          mbar_wait(&o_bar[x], (uint32_t)((nkx - 1) & 1), p.flags)) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int64_t qrow = (int64_t)q_begin + t_local;
        const int h = g * G + (r % G);
        __nv_bfloat16* dst = p.out + (qrow * p.num_q_heads + h) * D;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + colO + c, o);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack_bf16(o[i] * inv, o[i + 1] * inv);
              v.y = pack_bf16(o[i + 2] * inv, o[i + 3] * inv);
              v.z = pack_bf16(o[i + 4] * inv, o[i + 5] * inv);
              v.w = pack_bf16(o[i + 6] * inv, o[i + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c + i) = v;
            }
          }
        }
        if (row_ok && p.lse)
          p.lse[qrow * p.num_q_heads + h] =
              l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kProducerWarp) {
    // no bulk copy may still be landing in shared memory when the CTA exits
    for (int j = max(0, n_kv - kStages); j < n_kv; ++j) {
      mbar_wait(&k_full[j % kStages], (uint32_t)((j / kStages) & 1), p.flags);
      mbar_wait(&v_full[j % kStages], (uint32_t)((j / kStages) & 1), p.flags);
    }
  }
  if (warp == kMmaWarp) {
    mbar_wait(done_bar, 0, p.flags);
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int kFmt>
size_t smem_bytes() {
  return 1024 + Smem<D, kFmt>::kBytes + (20 + kFactsRing) * sizeof(uint64_t) +
         kFactsRing * sizeof(TileFacts) + 32;  // + TMEM base and the item
}

template <int D, int kFmt>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const Params& p, cudaStream_t stream) {
  const size_t smem = smem_bytes<D, kFmt>();
  // The shared-memory attribute belongs to the current device: set it once
  // per device and instantiation.
  constexpr int kMaxDevices = 64;
  static bool attr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr[dev]) {
      e = cudaFuncSetAttribute(prefill_kernel<D, kFmt>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr[dev] = true;
    }
  }
  const unsigned blocks = (unsigned)p.pair_slots * (unsigned)p.num_kv_heads * (unsigned)p.num_chunks;
  prefill_kernel<D, kFmt><<<blocks, Smem<D, kFmt>::kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace pf

// 3-D view of the packed queries [total_q][Hq][D] with a [128/G][G][64] box.
static int encode_q_map(CUtensorMap* map, const void* q, int total_q, int hq, int d, int group);

int prefill_entry(const pkv_cache* cache, const void* q, int32_t num_q_heads, int32_t gqa_group,
                  const int32_t* cu_q_lens, const int32_t* page_table, int32_t max_pages_per_seq,
                  const int32_t* seq_lens, int32_t num_chunks, int32_t total_q,
                  int32_t max_q_len, float softmax_scale, void* out, float* lse,
                  cudaStream_t stream) {
  int st = check_cache(cache);
  if (st) return st;
  if ((st = check_group(cache, num_q_heads, gqa_group))) return st;
  if (num_chunks < 0 || total_q < 0 || max_q_len < 0 || max_pages_per_seq < 1)
    return PKV_ERR_SHAPE;
  if ((st = check_table_span(cache, max_pages_per_seq))) return st;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PKV_ERR_SHAPE;
  if (num_chunks == 0 || total_q == 0 || max_q_len == 0) return PKV_OK;
  if (!q || !cu_q_lens || !page_table || !seq_lens || !out) return PKV_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
    return PKV_ERR_ALIGN;
  const int fmt = cache->kv_dtype;
  const int D = cache->head_dim;
  CUtensorMap tq, tk, tv;
  if ((st = encode_q_map(&tq, q, total_q, num_q_heads, D, gqa_group))) return st;
  const int64_t rows = (int64_t)cache->num_pages * cache->num_kv_heads * cache->page_size;
  // bf16 pools: 64-column boxes; quantised pools: one box of the whole row of
  // codes (D bytes, or D/2 for FP4)
  const bool bytes = quant(fmt);
  const int row_elems = fp4(fmt) ? D / 2 : D;
  const int box_cols = bytes ? row_elems : 64;
  if ((st = encode_pool_map(&tk, cache->k_pool, bytes, rows, row_elems, box_cols, 64))) return st;
  if ((st = encode_pool_map(&tv, cache->v_pool, bytes, rows, row_elems, box_cols, 64))) return st;
  pf::Params p;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  p.k_blocks = fp4(fmt) ? static_cast<const uint8_t*>(cache->k_pool) + block_region_offset(cache)
                        : nullptr;
  p.v_blocks = fp4(fmt) ? static_cast<const uint8_t*>(cache->v_pool) + block_region_offset(cache)
                        : nullptr;
  p.cu_q = cu_q_lens;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.flags = cache->error_flags;
  p.num_chunks = num_chunks;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = cache->num_kv_heads;
  p.group = gqa_group;
  p.max_pages = max_pages_per_seq;
  p.num_pages = cache->num_pages;
  p.page_size = cache->page_size;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  const int pair_tokens = 2 * (pf::kRows / gqa_group);  // two Q tiles per CTA
  p.pair_slots = (max_q_len + pair_tokens - 1) / pair_tokens;
  p.lpt = num_chunks <= pf::kLptMaxChunks ? 1 : 0;
  if ((int64_t)p.pair_slots * p.num_kv_heads * num_chunks > INT32_MAX) return PKV_ERR_SHAPE;
  cudaError_t e;
  if (D == 128)
    e = fmt == PKV_KV_NVFP4      ? pf::launch<128, PKV_KV_NVFP4>(tq, tk, tv, p, stream)
        : fmt == PKV_KV_INT8     ? pf::launch<128, PKV_KV_INT8>(tq, tk, tv, p, stream)
        : fmt == PKV_KV_FP8_E4M3 ? pf::launch<128, PKV_KV_FP8_E4M3>(tq, tk, tv, p, stream)
                                 : pf::launch<128, PKV_KV_BF16>(tq, tk, tv, p, stream);
  else
    e = fmt == PKV_KV_NVFP4      ? pf::launch<64, PKV_KV_NVFP4>(tq, tk, tv, p, stream)
        : fmt == PKV_KV_INT8     ? pf::launch<64, PKV_KV_INT8>(tq, tk, tv, p, stream)
        : fmt == PKV_KV_FP8_E4M3 ? pf::launch<64, PKV_KV_FP8_E4M3>(tq, tk, tv, p, stream)
                                 : pf::launch<64, PKV_KV_BF16>(tq, tk, tv, p, stream);
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFnQ)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int encode_q_map(CUtensorMap* map, const void* q, int total_q, int hq, int d, int group) {
  void* fnp = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fnp, cudaEnableDefault, &qr) !=
          cudaSuccess ||
      qr != cudaDriverEntryPointSuccess || !fnp)
    return PKV_ERR_CUDA;
  EncodeTiledFnQ fn = reinterpret_cast<EncodeTiledFnQ>(fnp);
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)hq, (cuuint64_t)total_q};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)hq * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(pf::kRows / group)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
