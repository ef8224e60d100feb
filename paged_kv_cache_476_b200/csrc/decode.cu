// Split-KV decode attention over a paged KV cache (sm_100a).
//
// What it computes (TensorRT-LLM concept page, "執行時執行模型": every step the
// attention operator reads the KV pages; "PagedAttention 及 KV 快取管理": pages
// are found through a per-sequence page table): for each sequence b and q head
// h, out = softmax(scale * q K_b^T) V_b over the seq_lens[b] cached tokens.
//
// Design (B200-first, HBM-bound):
//  * Work list.  Each (sequence, kv head) pair is a unit; a unit's tokens are
//    cut into tiles (64 tokens for bf16 and FP4 pools, 128 for one-byte
//    codes, so that a tile is 32 KB of K and V in either case).  The units'
//    tiles, concatenated in (b, g) order, are split into C equal contiguous
//    ranges, one per CTA, with C = SMs x resident CTAs per SM: one
//    persistent wave, no tail of unequal splits.
//  * A range cuts a unit into segments.  A segment computes an online-softmax
//    partial (m, l, unnormalised o) for the unit's G = Hq/Hkv q heads.  A
//    segment that covers its whole unit writes the output directly; otherwise
//    it stores its partial, and a small merge kernel (a programmatic
//    dependent launch, one warp per unit) combines the pieces afterwards.
//  * Warp roles: one producer warp walks the range and issues TMA loads of
//    the K and V tile (page-table indirected, one 64-row box per page and
//    box column, swizzled) into a multi-stage mbarrier ring, plus a bulk copy
//    of Q at each segment start; four consumer warps each take a quarter of
//    the tile's tokens and run S = Q K^T and O^T += V^T P^T on mma.sync, with
//    the online softmax in registers; a flush warp turns the consumers'
//    snapshots at each segment end into the output or a split partial while
//    the consumers stream on.
//  * Quantised K/V: INT8 K codes feed the s8 MMA (k = 32) as they land,
//    against a two-term fixed-point Q; E4M3 K and all V codes convert
//    exactly to f16 in registers after ldmatrix (FP4 times its E4M3 block
//    scales).  The per-(page, head) scales fold into the scores (K) and
//    into P (V).
//  * Every wait is bounded; a bad page id or length is skipped and flagged.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace pkv {

constexpr int kConsumerWarps = 4;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kFlushWarp = kConsumerWarps + 1;
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kMaxGroup = 8;
constexpr int kBoxRows = 64;   // rows of one TMA box; a tile is one or two of them
// Suspend hints (ns) of the waits: the flush warp idles for long stretches.
#ifndef PKV_FLUSH_SLEEP_NS
#define PKV_FLUSH_SLEEP_NS 20000
#endif
#ifndef PKV_PIPE_SLEEP_NS
#define PKV_PIPE_SLEEP_NS 0
#endif

// TileInfo.flags
constexpr int kSegFirst = 1;   // first tile of a segment: reset state, Q in this stage
constexpr int kSegLast = 2;    // last tile of a segment: flush after it
constexpr int kUnitWhole = 4;  // the segment is the whole unit: write out directly
constexpr int kBadHalf = 8;    // kBadHalf << h: the page of 64-row half h is invalid, skipped


struct TileInfo {
  int32_t b, g, tile, valid;  // valid = tokens of this tile below the length
  int32_t flags;
  int32_t slot;      // partial slot of this CTA's segment
  int32_t seg_base;  // first partial slot of the unit
  int32_t nseg;      // segments of the unit
  float ks[2], vs[2];  // scales of the pages of the tile's 64-row halves
};

// What the consumers hand to the flush warp at the end of a segment.
struct FlushDesc {
  int32_t b, g, slot, seg_base, nseg, whole, final;
};

template <int D, int kFmt>
struct Layout {
  // One-byte codes: 128-token tiles, 32 tokens per consumer warp, so that a
  // stage carries as many bytes as a bf16 one and a warp's work per barrier
  // doubles.  bf16 and FP4: 64-token tiles, 16 tokens per warp.
  static constexpr bool kWide = k8(kFmt);
  static constexpr int kTile = kWide ? 128 : 64;
  static constexpr int kHalves = kTile / kBoxRows;  // 64-row boxes (pages) per tile
  static constexpr int kWarpTok = kTile / kConsumerWarps;
  static constexpr int kMapEB = kFmt == PKV_KV_BF16 ? 2 : 1;   // element bytes of the TMA map
  static constexpr int kRowB = row_code_bytes(kFmt, D);        // code bytes of a token row
  static constexpr int kBoxRowB = kRowB >= 128 ? 128 : kRowB;  // TMA box inner bytes
  static constexpr int kNumBox = kRowB / kBoxRowB;             // boxes per tile row
  static constexpr int kBoxB = kTile * kBoxRowB;               // one box column of the tile
  static constexpr int kTileB = kNumBox * kBoxB;  // codes of one K (or V) tile
  // FP4: the E4M3 block scales of a tile's rows, after the two code tiles
  static constexpr int kScaleRowB = row_scale_bytes(kFmt, D);
  static constexpr int kScaleB = kTile * kScaleRowB;
  static constexpr int kStageB = 2 * kTileB + 2 * kScaleB;
  // bytes of one 64-row half of a stage (K and V, codes and block scales)
  static constexpr int kHalfTx = 2 * kNumBox * kBoxRows * kBoxRowB + 2 * kBoxRows * kScaleRowB;
};

// Shared-memory carve-up; the Q slices and the reduction buffers are sized
// by the GQA group so that two CTAs fit on one SM.  kSnap snapshot slots:
// one per consumer warp (4), or one per warp pair (2) where that buys a
// deeper ring.
struct SmemPlan {
  uint32_t q, red_o, red_m, red_l, bars, info, misc, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int D, int kFmt, int kStages, int kSnap>
__host__ __device__ inline SmemPlan smem_plan(int G) {
  using Ly = Layout<D, kFmt>;
  SmemPlan s;
  uint32_t o = kStages * Ly::kStageB;
  s.q = o;
  o += kStages * align_up(G * D * 2, 128);
  o = align_up(o, 1024);
  s.red_o = o;
  o += kSnap * G * (D + 4) * 4;  // rows padded by 4 floats (no bank conflicts)
  s.red_m = o;
  o += kSnap * G * 4;
  s.red_l = o;
  o += kSnap * G * 4;
  o = align_up(o, 8);
  s.bars = o;
  o += (2 * kStages + 3) * 8;
  s.info = o;
  o += kStages * sizeof(TileInfo) + sizeof(FlushDesc);
  s.misc = o;
  o += 2 * sizeof(int32_t);
  s.total = o;
  return s;
}

// Byte addresses in a TMA-swizzled tile made of kNumBox boxes of
// [rows][kBoxRowB]: chunk c (16 bytes) of row r lies at box (c / chunks per
// box), row offset r * kBoxRowB, chunk (c % chunks per box) XOR the row bits
// of the swizzle (128-, 64- or 32-byte pattern).
// Each lane's address is split into its own part, computed once, and a part
// known at compile time.  A lane reads chunk ce + lo of row `row` for even
// chunks ce; with xk the row bits the swizzle XORs into the chunk index,
// (ce + lo) ^ xk = (ce ^ (xk & ~1)) + (lo ^ (xk & 1)), so the address is
// base + box(ce) + a + ((ce % chunks-per-box) * 16 ^ x).  Rows 16 apart share
// the swizzle phase, so a lane tile moved by 16 rows is the base moved by
// 16 * kBoxRowB bytes.
struct LaneTile {
  uint32_t a;  // row * box row bytes + 16 * (lo ^ (xk & 1))
  uint32_t x;  // 16 * (xk & ~1)
};

template <int kBoxRowB>
__device__ __forceinline__ LaneTile lane_tile(int row, int lo) {
  constexpr int kShift = kBoxRowB == 128 ? 0 : kBoxRowB == 64 ? 1 : 2;
  constexpr int kMask = kBoxRowB / 16 - 1;
  const int xk = (row >> kShift) & kMask;
  return {(uint32_t)(row * kBoxRowB + ((lo ^ (xk & 1)) << 4)), (uint32_t)((xk & ~1) << 4)};
}

template <int kBoxRowB, int kRows>
__device__ __forceinline__ uint32_t tile_at(uint32_t base, LaneTile lt, int ce) {
  constexpr int kChunksPerBox = kBoxRowB / 16;
  return base + (ce / kChunksPerBox) * (kRows * kBoxRowB) + lt.a +
         (((uint32_t)(ce % kChunksPerBox) << 4) ^ lt.x);
}

// CTA (of C <= T over T virtual tiles) whose range [c*T/C, (c+1)*T/C) holds
// virtual tile x.  With C <= T every range is non-empty.
__device__ __forceinline__ int64_t cta_of(int64_t x, int64_t C, int64_t T) {
  return ((x + 1) * C - 1) / T;
}

template <int kTile>
__device__ __forceinline__ int tiles_of(int32_t len) { return (len + kTile - 1) / kTile; }

__device__ __forceinline__ int32_t clamp_len(const DecodeParams& p, int32_t len, bool report) {
  const int32_t cap = p.max_pages * p.page_size;
  if (len < 0 || len > cap) {
    if (report) flag_error(p.flags, PKV_FLAG_BAD_LENGTH);
    return len < 0 ? 0 : cap;
  }
  return len;
}

// The work list counts each unit as its tiles plus kCost virtual tiles after
// them, which load nothing: they stand for what a unit end costs the
// consumers (a segment hand-off, and on average half a tile of idle lanes),
// so that the equal split hands fewer real tiles to ranges in which many
// short units end.  Quantised pools, whose consumers bound the call, count
// one; bf16 pools, bound by HBM (a unit end hides under the tile waits),
// count none.
template <int kFmt>
__host__ __device__ constexpr int unit_end_cost() { return quant(kFmt) ? 1 : 0; }

// The first real tile at or after virtual index v: sequence b, kv head g,
// tile t, its virtual index xv and its real index (real tiles before it).
// Past the last tile, b = batch and (xv, real) are the totals.  Warp-wide.
struct TilePos {
  int b, g, t;
  int64_t xv, real;
};

template <int kTile, int kCost>
__device__ TilePos locate_tile(const DecodeParams& p, int64_t v, int lane) {
  const int Hkv = p.num_kv_heads;
  int64_t run_v = 0, run_r = 0;
  for (int base = 0; base < p.batch; base += 32) {
    const int b = base + lane;
    const int t = b < p.batch ? tiles_of<kTile>(clamp_len(p, __ldg(p.seq_lens + b), false)) : 0;
    const int vt = t > 0 ? t + kCost : 0;  // virtual tiles of one unit of b
    int incl_v = vt, incl_r = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yv = __shfl_up_sync(0xffffffffu, incl_v, o);
      const int yr = __shfl_up_sync(0xffffffffu, incl_r, o);
      if (lane >= o) {
        incl_v += yv;
        incl_r += yr;
      }
    }
    const int chunk_v = __shfl_sync(0xffffffffu, incl_v, 31);
    const int chunk_r = __shfl_sync(0xffffffffu, incl_r, 31);
    if (run_v + (int64_t)chunk_v * Hkv > v) {
      const bool hit = run_v + (int64_t)incl_v * Hkv > v;
      const int l0 = __ffs(__ballot_sync(0xffffffffu, hit)) - 1;
      const int t0 = __shfl_sync(0xffffffffu, t, l0);
      const int vt0 = __shfl_sync(0xffffffffu, vt, l0);
      const int ev0 = __shfl_sync(0xffffffffu, incl_v - vt, l0);
      const int er0 = __shfl_sync(0xffffffffu, incl_r - t, l0);
      const int64_t off = v - (run_v + (int64_t)ev0 * Hkv);  // in [0, vt0 * Hkv)
      const int g = (int)(off / vt0);
      const int po = (int)(off - (int64_t)g * vt0);
      const int64_t unit_v = run_v + (int64_t)ev0 * Hkv + (int64_t)g * vt0;
      const int64_t unit_r = run_r + (int64_t)er0 * Hkv + (int64_t)g * t0;
      if (po < t0) return {base + l0, g, po, unit_v + po, unit_r + po};
      // v lies on the unit's end cost: the next unit's first tile (of the
      // next sequence with tiles, past the last kv head)
      TilePos r = {base + l0, g + 1, 0, unit_v + vt0, unit_r + t0};
      if (r.g == Hkv) {
        r.g = 0;
        do {
          ++r.b;
        } while (r.b < p.batch && tiles_of<kTile>(clamp_len(p, __ldg(p.seq_lens + r.b), false)) == 0);
      }
      return r;
    }
    run_v += (int64_t)chunk_v * Hkv;
    run_r += (int64_t)chunk_r * Hkv;
  }
  return {p.batch, 0, 0, run_v, run_r};
}

// Fused append: the producer warp writes sequence b's newest token (K and V
// of kv head g, from k_new/v_new [B][Hkv][D]) into pool row (pid, g, slot):
// the bytes paged_kv_append writes for it (bf16 bits, or the one-byte codes
// of the quotient by the page's scale).  Four values per lane.
template <int D, int kFmt>
__device__ __forceinline__ void append_newest(const DecodeParams& p, int b, int g, int pid,
                                              int slot, float ks, float vs, int lane) {
  const int64_t src = ((int64_t)b * p.num_kv_heads + g) * D;
  const int64_t dst = (((int64_t)pid * p.num_kv_heads + g) * p.page_size + slot) * D;
  if constexpr (fp4(kFmt)) {
    // lanes 0..D/16-1 quantise K's blocks, lanes 16..16+D/16-1 V's
    const int blk = lane & 15;
    const bool is_v = lane >= 16;
    if (blk < D / 16) {
      const uint4* x = reinterpret_cast<const uint4*>((is_v ? p.v_new : p.k_new) + src + blk * 16);
      uint32_t sb;
      const uint2 codes = nvfp4_encode_block(x[0], x[1], is_v ? vs : ks, &sb);
      const int64_t row = dst / D;
      *reinterpret_cast<uint2*>((is_v ? p.v_pool : p.k_pool) + row * (D / 2) + blk * 8) = codes;
      (is_v ? p.v_blocks_w : p.k_blocks_w)[row * (D / 16) + blk] = static_cast<uint8_t>(sb);
    }
  } else {
    for (int e = lane * 4; e < D; e += 128) {
      const uint2 kx = *reinterpret_cast<const uint2*>(p.k_new + src + e);
      const uint2 vx = *reinterpret_cast<const uint2*>(p.v_new + src + e);
      if constexpr (!k8(kFmt)) {
        *reinterpret_cast<uint2*>(p.k_pool + (dst + e) * 2) = kx;
        *reinterpret_cast<uint2*>(p.v_pool + (dst + e) * 2) = vx;
      } else {
        auto codes = [](uint2 x, float s) -> uint32_t {
          const uint32_t lo = encode8x2<kFmt>(*reinterpret_cast<const __nv_bfloat162*>(&x.x), s);
          const uint32_t hi = encode8x2<kFmt>(*reinterpret_cast<const __nv_bfloat162*>(&x.y), s);
          return lo | (hi << 16);
        };
        *reinterpret_cast<uint32_t*>(p.k_pool + dst + e) = codes(kx, ks);
        *reinterpret_cast<uint32_t*>(p.v_pool + dst + e) = codes(vx, vs);
      }
    }
  }
}

template <int D, int kFmt, int kStages, int kSnap>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using Ly = Layout<D, kFmt>;
  constexpr int kTile = Ly::kTile;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte align the dynamic window (the swizzle pattern needs it).
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int G = p.group;
  const SmemPlan sp = smem_plan<D, kFmt, kStages, kSnap>(G);
  const uint32_t kQStride = align_up(G * D * 2, 128);
  constexpr int kRedRow = D + 4;  // row stride (floats) of the snapshot buffers
  uint8_t* tiles = smem;
  uint8_t* qbuf = smem + sp.q;
  float* red_o = reinterpret_cast<float*>(smem + sp.red_o);
  float* red_m = reinterpret_cast<float*>(smem + sp.red_m);
  float* red_l = reinterpret_cast<float*>(smem + sp.red_l);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sp.bars);
  uint64_t* empty = full + kStages;
  uint64_t* red_full = empty + kStages;   // consumers -> flush warp: the kSnap snapshots are ready
  uint64_t* red_empty = red_full + 1;     // flush warp -> consumers: snapshots consumed
  uint64_t* pair_full = red_empty + 1;    // (kSnap 2) warps 2, 3 -> warps 0, 1: written
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + sp.info);
  FlushDesc* desc = reinterpret_cast<FlushDesc*>(info + kStages);
  int32_t* s_misc = reinterpret_cast<int32_t*>(smem + sp.misc);  // [0]=n tiles, [1]=is_last

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int Hkv = p.num_kv_heads;
  // The merge kernel that follows waits for this grid's completion itself;
  // letting it launch now hides its launch latency behind this kernel.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t C = gridDim.x;
  const int64_t c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init(red_full, kSnap);
    mbar_init(red_empty, 1);
    if (kSnap < kConsumerWarps) mbar_init(pair_full, kConsumerWarps - kSnap);
    fence_barrier_init();
  }

  // ------------------------------------------------ producer: plan + loads
  int64_t n_tiles = 0;
  int pb = 0, pg = 0, pt = 0;  // producer's position (b, g, tile) at the range start
  int64_t range_start = 0, T = 0, Ce = 1;
  if (warp == kProducerWarp) {
    // Total virtual tiles over all units (real tiles plus the end costs).
    int64_t tot = 0;
    for (int base = 0; base < p.batch; base += 32) {
      const int b = base + lane;
      const int t = b < p.batch ? tiles_of<kTile>(clamp_len(p, __ldg(p.seq_lens + b), c == 0)) : 0;
      tot += t > 0 ? t + unit_end_cost<kFmt>() : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    T = tot * Hkv;
    // Only min(C, T) CTAs take work.  A range may hold only end costs (no
    // real tile); a unit's segment count is the number of ranges that hold
    // its real tiles, and every range between its first and last holds some.
    Ce = C < T ? C : T;
    if (c < Ce) {
      constexpr int kCost = unit_end_cost<kFmt>();
      const TilePos s0 = locate_tile<kTile, kCost>(p, (c * T) / Ce, lane);
      const TilePos s1 = locate_tile<kTile, kCost>(p, ((c + 1) * T) / Ce, lane);
      n_tiles = s1.real - s0.real;
      pb = s0.b;
      pg = s0.g;
      pt = s0.t;
      range_start = s0.xv;  // virtual index of the range's first real tile
    }
    // Empty sequences (length 0): out = 0, lse = -inf, written by one CTA each.
    for (int b = (int)((c * p.batch) / C); b < (int)(((c + 1) * p.batch) / C); ++b) {
      if (clamp_len(p, __ldg(p.seq_lens + b), false) == 0) {
        for (int i = lane; i < p.num_q_heads * D; i += 32)
          p.out[(int64_t)b * p.num_q_heads * D + i] = __float2bfloat16(0.f);
        if (p.lse)
          for (int h = lane; h < p.num_q_heads; h += 32)
            p.lse[(int64_t)b * p.num_q_heads + h] = -INFINITY;
      }
    }
    if (lane == 0) s_misc[0] = (int)n_tiles;
  }
  __syncthreads();
  n_tiles = s_misc[0];
  if (n_tiles == 0) return;

  if (warp == kFlushWarp) {
    // ---------------------------------------------------------- flush warp
    // Turns each segment's kSnap snapshots into the output (whole unit) or a
    // split partial.  It overlaps the consumers, which keep streaming the
    // next segment.
    for (int k = 0;; ++k) {
      if (!mbar_wait(red_full, (uint32_t)(k & 1), p.flags, PKV_FLUSH_SLEEP_NS)) return;
      const FlushDesc fd = *desc;
      for (int r = 0; r < G; ++r) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kSnap; ++w) M = fmaxf(M, red_m[w * G + r]);
        float sc[kSnap];
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < kSnap; ++w) {
          const float mw = red_m[w * G + r];
          sc[w] = (M == -INFINITY || mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
          den += sc[w] * red_l[w * G + r];
        }
        const int64_t orow = (int64_t)fd.b * p.num_q_heads + fd.g * G + r;
        const float inv = den > 0.f ? 1.f / den : 0.f;
        // four consecutive d per lane: 16-byte snapshot reads, one 8-byte
        // (bf16 output) or 16-byte (partial) store
        for (int d0 = 4 * lane; d0 < D; d0 += 128) {
          float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w = 0; w < kSnap; ++w) {
            const float4 o = *reinterpret_cast<const float4*>(red_o + (w * G + r) * kRedRow + d0);
            num.x += sc[w] * o.x;
            num.y += sc[w] * o.y;
            num.z += sc[w] * o.z;
            num.w += sc[w] * o.w;
          }
          if (fd.whole) {
            uint2 packed;
            packed.x = pack_bf16(num.x * inv, num.y * inv);
            packed.y = pack_bf16(num.z * inv, num.w * inv);
            *reinterpret_cast<uint2*>(p.out + orow * D + d0) = packed;
          } else {
            *reinterpret_cast<float4*>(p.part_o + ((int64_t)fd.slot * G + r) * D + d0) = num;
          }
        }
        if (lane == 0) {
          if (fd.whole) {
            if (p.lse) p.lse[orow] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
          } else {
            p.part_ml[(int64_t)fd.slot * G + r] = make_float2(M, den);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(red_empty);  // the snapshot buffers are free again
      if (fd.final) return;
    }
  }

  if (warp == kProducerWarp) {
    // ------------------------------------------------------ producer loop
    const uint64_t pol = policy_evict_first();
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
    }
    const int P = p.page_size;
    int b = pb, g = pg, t = pt;
    int len = clamp_len(p, __ldg(p.seq_lens + b), false);
    int ntile = tiles_of<kTile>(len);
    int seg_first_t = t;
    // page ids (and scales) of 32 consecutive pages, one per lane
    int cache_key = -1, cache_j0 = 0;
    int my_pid = 0;
    float my_ks = 1.f, my_vs = 1.f;
    int64_t x = range_start;  // virtual index of the tile at hand
    int u_seg_base = 0, u_nseg = 1, u_slot = 0;
    int issued = 0;
    for (int64_t i = 0; i < n_tiles; ++i, ++x) {
      const int stage = (int)(i % kStages);
      if (i >= kStages) {
        if (!mbar_wait(&empty[stage], (uint32_t)((i / kStages - 1) & 1), p.flags,
                       PKV_PIPE_SLEEP_NS))
          break;
      }
      // A tile is kTile tokens from tok0, in 64-row halves; page sizes are
      // multiples of 64, so each half lies in one page.
      const int tok0 = t * kTile;
      const int pages_b = (len + P - 1) / P;
      const int j_first = tok0 / P;
      const int j_last = min((tok0 + kTile - 1) / P, pages_b - 1);
      const int key = quant(kFmt) ? b * Hkv + g : b;
      if (cache_key != key || j_first < cache_j0 || j_last >= cache_j0 + 32) {
        cache_key = key;
        cache_j0 = j_first;
        const int jj = j_first + lane;
        my_pid = jj < pages_b ? __ldg(p.page_table + (int64_t)b * p.max_pages + jj) : 0;
        if constexpr (quant(kFmt)) {
          if (jj < pages_b && my_pid >= 0 && my_pid < p.num_pages) {
            my_ks = __ldg(p.k_scale + (int64_t)my_pid * Hkv + g);
            my_vs = __ldg(p.v_scale + (int64_t)my_pid * Hkv + g);
          }
        }
      }
      int hpid[Ly::kHalves], hrow[Ly::kHalves], hflags = 0;
      bool hhas[Ly::kHalves];
      float hks[2] = {1.f, 1.f}, hvs[2] = {1.f, 1.f};
#pragma unroll
      for (int h = 0; h < Ly::kHalves; ++h) {
        const int tokh = tok0 + kBoxRows * h;
        hhas[h] = tokh < len;  // half 0 always: t < ntile
        const int jh = min(tokh / P, pages_b - 1);
        hrow[h] = tokh - (tokh / P) * P;
        int pid = __shfl_sync(0xffffffffu, my_pid, jh - cache_j0);
        if constexpr (quant(kFmt)) {
          hks[h] = __shfl_sync(0xffffffffu, my_ks, jh - cache_j0);
          hvs[h] = __shfl_sync(0xffffffffu, my_vs, jh - cache_j0);
        }
        bool bad = pid < 0 || pid >= p.num_pages;
        if (bad && hhas[h] && lane == 0) flag_error(p.flags, PKV_FLAG_BAD_PAGE);
        if constexpr (quant(kFmt)) {
          if (!bad && !(hks[h] > 0.f && hks[h] <= 32768.f && hvs[h] > 0.f && hvs[h] <= 32768.f)) {
            bad = true;
            if (hhas[h] && lane == 0) flag_error(p.flags, PKV_FLAG_BAD_SCALE);
          }
        }
        if (bad) {
          pid = 0;
          hflags |= kBadHalf << h;
        }
        hpid[h] = pid;
      }
      // Fused append: this CTA is the one that reads the tile holding the
      // sequence's newest token (position len - 1), so it stores the token
      // first (as paged_kv_append would: whenever the page id is valid) and
      // orders those generic-proxy stores before its own bulk-tensor loads.
      if (p.k_new && t == ntile - 1 && __ldg(p.seq_lens + b) == len) {
        const int jn = (len - 1) / P;
        const int pid_n = __shfl_sync(0xffffffffu, my_pid, jn - cache_j0);
        if (pid_n >= 0 && pid_n < p.num_pages) {
          const int hn = (len - 1 - tok0) / kBoxRows;  // the half holding it (same page)
          append_newest<D, kFmt>(p, b, g, pid_n, (len - 1) % P, hn ? hks[1] : hks[0],
                                 hn ? hvs[1] : hvs[0], lane);
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        __syncwarp();
      }
      const bool first = (i == 0) || (t == 0);
      if (first) seg_first_t = t;
      const bool last = (i == n_tiles - 1) || (t == ntile - 1);
      if (lane == 0) {
        TileInfo ti;
        ti.b = b;
        ti.g = g;
        ti.tile = t;
        ti.valid = min(kTile, len - tok0);
        ti.flags = (first ? kSegFirst : 0) | (last ? kSegLast : 0) | hflags;
        if (last && seg_first_t == 0 && t == ntile - 1) ti.flags |= kUnitWhole;
        if (first) {
          // once per unit: which CTAs share it, hence its partial slots
          const int64_t u = (int64_t)b * Hkv + g;
          const int64_t x_unit = x - t;  // virtual index of the unit's first tile
          const int64_t c_first = cta_of(x_unit, Ce, T);
          const int64_t c_last = cta_of(x_unit + ntile - 1, Ce, T);
          u_seg_base = (int)(u + c_first);
          u_nseg = (int)(c_last - c_first + 1);
          u_slot = (int)(u + c);
          // the CTA holding the unit's first tile tells the merge kernel
          // where the unit's partials are (nseg == 1: written whole)
          if (t == 0) p.unit_info[u] = make_int2(u_seg_base, u_nseg);
        }
        ti.seg_base = u_seg_base;
        ti.nseg = u_nseg;
        ti.slot = u_slot;
        ti.ks[0] = hks[0];
        ti.vs[0] = hvs[0];
        ti.ks[1] = hks[1];
        ti.vs[1] = hvs[1];
        info[stage] = ti;
        const uint32_t qbytes = first ? (uint32_t)(G * D * 2) : 0u;
        uint32_t tx = qbytes;
#pragma unroll
        for (int h = 0; h < Ly::kHalves; ++h)
          if (hhas[h]) tx += Ly::kHalfTx;
        mbar_arrive_expect_tx(&full[stage], tx);
        uint8_t* kdst = tiles + stage * Ly::kStageB;
        uint8_t* vdst = kdst + Ly::kTileB;
#pragma unroll
        for (int h = 0; h < Ly::kHalves; ++h) {
          if (!hhas[h]) continue;
          const int32_t y = (int32_t)(((int64_t)hpid[h] * Hkv + g) * P + hrow[h]);
          const int hoff = h * kBoxRows * Ly::kBoxRowB;
#pragma unroll
          for (int bx = 0; bx < Ly::kNumBox; ++bx) {
            const int32_t xc = bx * (Ly::kBoxRowB / Ly::kMapEB);
            tma_load_2d(kdst + bx * Ly::kBoxB + hoff, &tmap_k, xc, y, &full[stage], pol);
            tma_load_2d(vdst + bx * Ly::kBoxB + hoff, &tmap_v, xc, y, &full[stage], pol);
          }
          if constexpr (fp4(kFmt)) {
            // the half's block scales: 64 consecutive rows of the block-scale
            // region, one contiguous run
            const int64_t soff = (int64_t)y * Ly::kScaleRowB;
            const int sdst = h * kBoxRows * Ly::kScaleRowB;
            bulk_load(vdst + Ly::kTileB + sdst, p.k_blocks + soff, kBoxRows * Ly::kScaleRowB,
                      &full[stage]);
            bulk_load(vdst + Ly::kTileB + Ly::kScaleB + sdst, p.v_blocks + soff,
                      kBoxRows * Ly::kScaleRowB, &full[stage]);
          }
        }
        if (first) {
          const __nv_bfloat16* src = p.q + ((int64_t)b * p.num_q_heads + (int64_t)g * G) * D;
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
              "[%3];" ::"r"(smem_u32(qbuf + stage * kQStride)),
              "l"(reinterpret_cast<uint64_t>(src)), "r"(qbytes), "r"(smem_u32(&full[stage]))
              : "memory");
        }
      }
      __syncwarp();
      ++issued;
      // advance to the next tile of the work list (past the unit's end cost)
      if (++t == ntile) {
        t = 0;
        x += unit_end_cost<kFmt>();
        if (++g == Hkv) {
          g = 0;
          do {
            ++b;
          } while (b < p.batch && tiles_of<kTile>(clamp_len(p, __ldg(p.seq_lens + b), false)) == 0);
          if (b < p.batch) {
            len = clamp_len(p, __ldg(p.seq_lens + b), false);
            ntile = tiles_of<kTile>(len);
          }
        }
      }
    }
    // Drain: wait (bounded) until the last issued loads have landed, so no
    // bulk copy is in flight into this CTA's shared memory when it exits.
    const int64_t lo = issued > kStages ? issued - kStages : 0;
    for (int64_t k = lo; k < issued; ++k)
      mbar_wait(&full[k % kStages], (uint32_t)((k / kStages) & 1), p.flags);
    return;
  }

  // ---------------------------------------------------------- consumers
  constexpr int NG = Ly::kWarpTok / 16;  // 16-token groups in a warp's share of the tile
  const int gid = lane >> 2;   // row of the mma fragment = q head within the group
  const int tid4 = lane & 3;
  const int mat = lane >> 3;   // which 8x8 matrix this lane addresses in ldmatrix.x4
  const int mrow = lane & 7;
  const bool row_ok = gid < G;
  const int wrow = Ly::kWarpTok * warp;     // this warp's first row of the tile
  const int my_half = wrow / kBoxRows;      // the 64-row half (page) its rows lie in
  int nflush = 0;

  constexpr int KS = D / 16;  // k-steps of 16 over head_dim
  // Q as the B operand of S^T = K Q^T (column gid = head gid): two k halves
  // (f16 / bf16), or for INT8's k = 32 products the four bytes at d = 16kk +
  // 4*tid4 of the two terms of a split Q ([0] high, [1] low)
  uint32_t qa[KS][2];
  // O^T accumulators: PV runs as O^T = V^T P^T (M = head_dim, N = 8 heads).
  // ot[m][0..1] = O[heads 2*tid4, 2*tid4+1][d = 16m + gid], ot[m][2..3] the same at d + 8.
  float ot[D / 16][4];
  // running max and partial sum of heads 2*tid4 and 2*tid4 + 1 (the O^T
  // columns of this thread)
  float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
  float qk_mul = p.scale_log2;  // multiplier of head gid's raw scores into log2 units
  float hmul[2] = {p.scale_log2, p.scale_log2};  // the same for heads 2*tid4, 2*tid4 + 1
  // K rows a lane addresses in ldmatrix.x4: matrices (tokens 0-7, chunk ce),
  // (0-7, ce+1), (8-15, ce), (8-15, ce+1), the A fragments (a0, a2, a1, a3)
  // of S^T for one 16-token group
  const LaneTile ltk = lane_tile<Ly::kBoxRowB>(wrow + mrow + (mat >> 1) * 8, mat & 1);
  // FP4 V: transposed 16-bit loads, matrices (tokens 0-7, ce), (8-15, ce),
  // (0-7, ce+1), (8-15, ce+1)
  const LaneTile ltv = lane_tile<Ly::kBoxRowB>(wrow + mrow + (mat & 1) * 8, mat >> 1);
  // One-byte V: the 8-bit transposing load takes 16 row addresses per
  // 16x16 matrix (lanes 0-15: chunk ce, lanes 16-31: chunk ce + 1); row
  // position 4i + e holds token 2i + (e & 1) + 8 (e >> 1) of a 16-token
  // group, so that a thread's four rows are the f16 A fragment's token
  // columns (below)
  const int vrow = 2 * ((lane & 15) >> 2) + (lane & 1) + 8 * ((lane >> 1) & 1);
  const LaneTile ltb = lane_tile<Ly::kBoxRowB>(wrow + vrow, lane >> 4);

  for (int64_t i = 0; i < n_tiles; ++i) {
    const int stage = (int)(i % kStages);
    if (!mbar_wait(&full[stage], (uint32_t)((i / kStages) & 1), p.flags, PKV_PIPE_SLEEP_NS))
      return;
    // only what the tile's math needs lives in registers; the segment
    // bookkeeping is read from the (still unreleased) stage at hand-off
    const int t_flags = info[stage].flags;
    const int t_valid = info[stage].valid;
    const float t_ks = quant(kFmt) ? info[stage].ks[my_half] : 1.f;
    const float t_vs = quant(kFmt) ? info[stage].vs[my_half] : 1.f;
    const uint8_t* qs = qbuf + stage * kQStride;
    if (t_flags & kSegFirst) {
      m_run[0] = m_run[1] = -INFINITY;
      l_part[0] = l_part[1] = 0.f;
#pragma unroll
      for (int m = 0; m < D / 16; ++m) ot[m][0] = ot[m][1] = ot[m][2] = ot[m][3] = 0.f;
      if constexpr (!quant(kFmt)) {
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qs + gid * D * 2);
          qa[kk][0] = row_ok ? qrow[(16 * kk + 2 * tid4) / 2] : 0u;
          qa[kk][1] = row_ok ? qrow[(16 * kk + 8 + 2 * tid4) / 2] : 0u;
        }
        qk_mul = p.scale_log2;
      } else {
        // Q with a per-row power-of-two prescale, in the d order of the K
        // codes that ldmatrix delivers: qv[kk] holds d = 16kk + 4*tid4 +
        // {0..3} for one-byte codes.  E4M3 uses f16 Q against converted codes
        // (the fragment's k pair (2*tid4, +1) holds d = 16kk + 4*tid4 + {0,1}
        // and the pair (2*tid4+8, +9) holds + {2,3}).  INT8 feeds the s8 MMA
        // (k = 32), which takes from a thread the bytes d = 32kp + 4*tid4 +
        // {0..3} and + 16 of one row, that is qv[2kp] and qv[2kp+1].  FP4 (f16
        // Q): a 16-byte chunk c holds d = 32c..32c+31 and a thread's 4 bytes
        // are d = 32c + 8*tid4 + {0..7}; k-step 2c takes the first four of
        // them, k-step 2c+1 the last four.
        float amax = 0.f;
        float qv[KS][4];
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(qs) + gid * D;
          const int d0 = fp4(kFmt) ? 32 * (kk >> 1) + 8 * tid4 + 4 * (kk & 1) : 16 * kk + 4 * tid4;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qv[kk][e] = row_ok ? __bfloat162float(qrow[d0 + e]) : 0.f;
            amax = fmaxf(amax, fabsf(qv[kk][e]));
          }
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        // power-of-two prescale putting amax in [2^(top-1), 2^top): 2^14 for
        // f16 Q, 2^13 for the INT8 split
        constexpr int kTop = kFmt == PKV_KV_INT8 ? 13 : 14;
        int ex = 0;
        if (amax > 0.f) {
          frexpf(amax, &ex);  // amax < 2^ex
          ex = kTop - ex;     // amax * 2^ex < 2^kTop
          ex = max(-100, min(100, ex));
        }
        const float pre = ldexpf(1.f, ex);
        if constexpr (kFmt == PKV_KV_INT8) {
          // 13-bit fixed point q = round(x * pre), split as q = 128 hi + lo
          // with hi in [-64, 64] and lo in [0, 127]: two s8 operands whose s32
          // products with the codes are exact
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            uint32_t hi = 0, lo = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int qf = __float2int_rn(qv[kk][e] * pre);
              hi |= ((uint32_t)(qf >> 7) & 0xffu) << (8 * e);
              lo |= ((uint32_t)qf & 0x7fu) << (8 * e);
            }
            qa[kk][0] = hi;
            qa[kk][1] = lo;
          }
        } else {
          // f16 (E4M3, FP4)
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            qa[kk][0] = pack_f16(qv[kk][0] * pre, qv[kk][1] * pre);
            qa[kk][1] = pack_f16(qv[kk][2] * pre, qv[kk][3] * pre);
          }
        }
        qk_mul = p.scale_log2 * ldexpf(1.f, -ex);
        hmul[0] = __shfl_sync(0xffffffffu, qk_mul, 8 * tid4);      // lane of head 2*tid4
        hmul[1] = __shfl_sync(0xffffffffu, qk_mul, 8 * tid4 + 4);  // head 2*tid4 + 1
      }
    }

    // tokens of my share below the length (none when my half's page is bad)
    const int valid = (t_flags & (kBadHalf << my_half)) ? 0 : t_valid - wrow;
    if (valid > 0) {
      const uint32_t kbase = smem_u32(tiles + stage * Ly::kStageB);
      const uint32_t vbase = kbase + Ly::kTileB;
      // ---- S^T = K Q^T over my tokens: a 16-token group fills the 16 rows
      // of a product, the group's heads its 8 columns ----
      // st[g] = S^T at (token gid, head 2*tid4), (gid, 2*tid4+1), (gid+8,
      // 2*tid4), (gid+8, 2*tid4+1) of group g (tokens 16g..16g+15 of my share)
      float st[NG][4];
      if constexpr (kFmt == PKV_KV_INT8) {
        // INT8 codes are the A operand of the s8 MMA (k = 32) as they land,
        // the two terms of the split Q its B; S = 128 hi + lo exactly in s32
        int32_t sh[NG][4], sl[NG][4];
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) sh[g][e] = sl[g][e] = 0;
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            uint32_t r[4];
            ldsm_x4(tile_at<Ly::kBoxRowB, kTile>(kbase + g * 16 * Ly::kBoxRowB, ltk, 2 * kp),
                    r[0], r[1], r[2], r[3]);
            mma_s8_full(sh[g], r[0], r[2], r[1], r[3], qa[2 * kp][0], qa[2 * kp + 1][0]);
            mma_s8_full(sl[g], r[0], r[2], r[1], r[3], qa[2 * kp][1], qa[2 * kp + 1][1]);
          }
        }
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) st[g][e] = (float)(sh[g][e] * 128 + sl[g][e]);
      } else {
        // f16 / bf16 products, two accumulation chains per group (even / odd
        // k-steps)
        float s2[NG][4];
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) st[g][e] = s2[g][e] = 0.f;
        if constexpr (kFmt == PKV_KV_FP8_E4M3) {
          // E4M3 codes convert exactly to f16 after ldmatrix, four per call:
          // (lo, hi) of a register are the k pairs (2*tid4, +1) and
          // (2*tid4+8, +9) of its token, Q permuted the same way
#pragma unroll
          for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              uint32_t r[4];
              ldsm_x4(tile_at<Ly::kBoxRowB, kTile>(kbase + g * 16 * Ly::kBoxRowB, ltk, 2 * kp),
                      r[0], r[1], r[2], r[3]);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t l0, h0, l1, h1;
                kv8x4_to_f16x2<kFmt>(r[h], l0, h0);      // token gid, chunk 2kp + h
                kv8x4_to_f16x2<kFmt>(r[2 + h], l1, h1);  // token gid + 8
                mma_f16(h ? s2[g] : st[g], l0, l1, h0, h1, qa[2 * kp + h][0], qa[2 * kp + h][1]);
              }
            }
          }
        } else if constexpr (!quant(kFmt)) {
#pragma unroll
          for (int kk = 0; kk < KS; ++kk) {
            uint32_t r[4];
            ldsm_x4(tile_at<Ly::kBoxRowB, kTile>(kbase, ltk, 2 * kk), r[0], r[1], r[2], r[3]);
            mma_bf16((kk & 1) ? s2[0] : st[0], r[0], r[2], r[1], r[3], qa[kk][0], qa[kk][1]);
          }
        } else {
          // FP4 codes: a register of 4 bytes holds d = 32c + 8*tid4 + {0..7}
          // of one token, all in block 2c + tid4/2; its four f16x2 (exact),
          // each times the token's block scale (exact in f16), are that
          // token's A registers of k-steps 2c (bytes 0, 1) and 2c+1 (bytes 2, 3).
          const uint8_t* ksc = tiles + stage * Ly::kStageB + 2 * Ly::kTileB;
          uint32_t sk[2][Ly::kScaleRowB / 4];  // block scales of tokens gid and gid+8
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int w4 = 0; w4 < Ly::kScaleRowB / 4; ++w4)
              sk[n][w4] = *reinterpret_cast<const uint32_t*>(
                  ksc + (wrow + 8 * n + gid) * Ly::kScaleRowB + 4 * w4);
#pragma unroll
          for (int c = 0; c < D / 32; c += 2) {
            // matrices: (tokens 0-7, chunk c), (0-7, c+1), (8-15, c), (8-15, c+1)
            uint32_t r[4];
            ldsm_x4(tile_at<Ly::kBoxRowB, kTile>(kbase, ltk, c), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int cc = c + h;
              const uint32_t blk = 2 * cc + (tid4 >> 1);
              uint32_t f0[4], f1[4];
              e2m1x8_to_f16x2(r[h], f0);
              e2m1x8_to_f16x2(r[2 + h], f1);
              const uint32_t sb0 = e4m3_splat_f16x2(sk[0][blk >> 2], blk & 3);
              const uint32_t sb1 = e4m3_splat_f16x2(sk[1][blk >> 2], blk & 3);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                f0[k] = hmul2_u32(f0[k], sb0);
                f1[k] = hmul2_u32(f1[k], sb1);
              }
              mma_f16(st[0], f0[0], f1[0], f0[1], f1[1], qa[2 * cc][0], qa[2 * cc][1]);
              mma_f16(s2[0], f0[2], f1[2], f0[3], f1[3], qa[2 * cc + 1][0], qa[2 * cc + 1][1]);
            }
          }
        }
#pragma unroll
        for (int g = 0; g < NG; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) st[g][e] += s2[g][e];
      }
      // ---- online softmax per head (log2 domain): this thread holds heads
      // 2*tid4 (e even) and 2*tid4 + 1 (e odd) for tokens 16g + gid + 8(e/2);
      // the eight lanes of a head column reduce over their tokens ----
      const float mul0 = quant(kFmt) ? hmul[0] * t_ks : hmul[0];
      const float mul1 = quant(kFmt) ? hmul[1] * t_ks : hmul[1];
      float x[NG][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int g = 0; g < NG; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in = 16 * g + gid + 8 * (e >> 1) < valid;
          x[g][e] = in ? st[g][e] * ((e & 1) ? mul1 : mul0) : -INFINITY;
          if (e & 1)
            mx1 = fmaxf(mx1, x[g][e]);
          else
            mx0 = fmaxf(mx0, x[g][e]);
        }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);  // finite: valid > 0
      const float al0 = fast_exp2(m_run[0] - mn0), al1 = fast_exp2(m_run[1] - mn1);
      float pr[NG][4];
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        pr[g][0] = fast_exp2(x[g][0] - mn0);
        pr[g][1] = fast_exp2(x[g][1] - mn1);
        pr[g][2] = fast_exp2(x[g][2] - mn0);
        pr[g][3] = fast_exp2(x[g][3] - mn1);
        ps0 += pr[g][0] + pr[g][2];
        ps1 += pr[g][1] + pr[g][3];
      }
      l_part[0] = l_part[0] * al0 + ps0;
      l_part[1] = l_part[1] * al1 + ps1;
      m_run[0] = mn0;
      m_run[1] = mn1;
      // The factors belong to this thread's own O^T columns.  Once the
      // running max settles (most tiles), no head's factor moves.
      if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
        for (int m = 0; m < D / 16; ++m) {
          ot[m][0] *= al0;
          ot[m][1] *= al1;
          ot[m][2] *= al0;
          ot[m][3] *= al1;
        }
      }
      // ---- O^T += V^T P^T over my tokens (P^T: a transpose of P packed) ----
      // V rows past the length may hold anything (NaN): on a partial tile
      // they are zeroed in the fragments, so that 0 * NaN never reaches the
      // accumulator.  Full shares, nearly all, take the product without masks.
      {
        // products over 16-token groups: the packed pairs (token gid, heads
        // 2*tid4, +1) and (token gid + 8, ...) transposed are P^T's B
        // fragments (head gid; tokens 2*tid4, +1 and 8 + 2*tid4, +1)
#pragma unroll
        for (int hv = 0; hv < NG; ++hv) {
          const int vh = valid - 16 * hv;  // tokens of this group below the length
          if (hv > 0 && vh <= 0) break;
          uint32_t q0, q1;
          if constexpr (!quant(kFmt)) {
            q0 = pack_bf16(pr[hv][0], pr[hv][1]);
            q1 = pack_bf16(pr[hv][2], pr[hv][3]);
          } else {
            q0 = pack_f16(pr[hv][0] * t_vs, pr[hv][1] * t_vs);
            q1 = pack_f16(pr[hv][2] * t_vs, pr[hv][3] * t_vs);
          }
          const uint32_t pa0 = movmatrix_t(q0);
          const uint32_t pa2 = movmatrix_t(q1);
          const uint32_t gbase = vbase + hv * 16 * Ly::kBoxRowB;
          auto pv_product = [&](auto masked) {
            constexpr bool kMasked = decltype(masked)::value;
            uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
            if constexpr (kMasked) {
              vm0 = (2 * tid4 < vh ? 0x0000ffffu : 0u) | (2 * tid4 + 1 < vh ? 0xffff0000u : 0u);
              vm1 = (2 * tid4 + 8 < vh ? 0x0000ffffu : 0u) | (2 * tid4 + 9 < vh ? 0xffff0000u : 0u);
            }
            // tokens 2*tid4, 2*tid4+1 (m0) or 2*tid4+8, 2*tid4+9 (m1) of a fragment
            auto m0 = [&](uint32_t a) -> uint32_t { return kMasked ? (a & vm0) : a; };
            auto m1 = [&](uint32_t a) -> uint32_t { return kMasked ? (a & vm1) : a; };
            if constexpr (!quant(kFmt)) {
#pragma unroll
              for (int m = 0; m < D / 16; ++m) {
                // A = V^T rows d 16m..16m+15: matrices (tokens 0-7, chunk 2m), (0-7, 2m+1),
                // (8-15, 2m), (8-15, 2m+1), transposed on load
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(tile_at<Ly::kBoxRowB, kTile>(gbase, ltk, 2 * m), a0, a1, a2, a3);
                mma_bf16(ot[m], m0(a0), m0(a1), m1(a2), m1(a3), pa0, pa2);
              }
            } else if constexpr (fp4(kFmt)) {
              // FP4 V codes from the landed tile.  A transposed load of 16-bit
              // elements (byte pairs) gives each thread, per 8x8 matrix, tokens
              // (2*tid4, 2*tid4+1) x codes d = 32c + 4*gid + {0..3} (low half:
              // the first token).  Interleaving the two tokens' nibbles makes
              // four bytes, one per d, each the token pair of that d, which
              // convert exactly to f16x2; times the two tokens' block scales
              // (block 2c + gid/4) they are the A fragments of V^T.  Fragment
              // rows: m-tile 2c holds d = 32c + 4*gid + {0, 1} (rows gid, gid+8),
              // m-tile 2c+1 holds d = 32c + 4*gid + {2, 3}; the snapshot below
              // undoes the order.
              const uint8_t* vsc = tiles + stage * Ly::kStageB + 2 * Ly::kTileB + Ly::kScaleB;
              uint32_t sv[4][Ly::kScaleRowB / 4];  // tokens 2t, 2t+1, 2t+8, 2t+9 of the warp
#pragma unroll
              for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int w4 = 0; w4 < Ly::kScaleRowB / 4; ++w4)
                  sv[k][w4] = *reinterpret_cast<const uint32_t*>(
                      vsc + (wrow + 2 * tid4 + (k & 1) + 8 * (k >> 1)) * Ly::kScaleRowB + 4 * w4);
              auto v_pairs = [&](uint32_t codes, uint32_t scale_pair, uint32_t* f) {
                const uint32_t x = __byte_perm(codes, 0u, 0x3120);  // A.d01 B.d01 A.d23 B.d23
                const uint32_t lo = x & 0x0f0f0f0fu;                // A.d0 B.d0 A.d2 B.d2
                const uint32_t hi = (x >> 4) & 0x0f0f0f0fu;         // A.d1 B.d1 A.d3 B.d3
                const uint32_t z = __byte_perm(lo | (lo >> 4), hi | (hi >> 4), 0x6240);
                e2m1x8_to_f16x2(z, f);                              // pairs of d0, d1, d2, d3
#pragma unroll
                for (int k = 0; k < 4; ++k) f[k] = hmul2_u32(f[k], scale_pair);
              };
#pragma unroll
              for (int c = 0; c < D / 32; c += 2) {
                // matrices: (tokens 0-7, chunk c), (8-15, c), (0-7, c+1), (8-15, c+1)
                uint32_t r0, r1, r2, r3;
                ldsm_x4_t(tile_at<Ly::kBoxRowB, kTile>(vbase, ltv, c), r0, r1, r2, r3);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int cc = c + h;
                  const uint32_t blk = 2 * cc + (gid >> 2);
                  const uint32_t s01 =
                      e4m3_pair_f16x2(sv[0][blk >> 2], blk & 3, sv[1][blk >> 2], blk & 3);
                  const uint32_t s89 =
                      e4m3_pair_f16x2(sv[2][blk >> 2], blk & 3, sv[3][blk >> 2], blk & 3);
                  uint32_t pf[4], qf[4];
                  v_pairs(h ? r2 : r0, s01, pf);  // tokens 2t, 2t+1
                  v_pairs(h ? r3 : r1, s89, qf);  // tokens 2t+8, 2t+9
                  mma_f16(ot[2 * cc], m0(pf[0]), m0(pf[1]), m1(qf[0]), m1(qf[1]), pa0, pa2);
                  mma_f16(ot[2 * cc + 1], m0(pf[2]), m0(pf[3]), m1(qf[2]), m1(qf[3]), pa0, pa2);
                }
              }
            } else {
              // One-byte V codes straight from the landed tile.  The transposing
              // load of 8-bit elements gives the thread (gid, tid4), for byte
              // column gid of a 16-byte chunk m (d = 16m + gid) and for column
              // gid + 8, the codes of rows 4*tid4 .. 4*tid4+3, which the row
              // order above makes tokens 2t, 2t+1, 2t+8, 2t+9 (t = tid4).  Two
              // exact conversions per register then give the A fragment of V^T
              // (rows d = 16m + gid and + 8, as in the bf16 path) with no byte
              // shuffles.
#pragma unroll
              for (int m = 0; m < D / 16; m += 2) {
                uint32_t r[4];  // chunk m: r[0] (column gid), r[1] (gid + 8); chunk m+1: r[2], r[3]
                ldsm_x2_t_b8(tile_at<Ly::kBoxRowB, kTile>(gbase, ltb, m), r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  uint32_t a0, a1, a2, a3;
                  kv8x4_to_f16x2<kFmt>(r[2 * h], a0, a2);      // d = 16(m+h) + gid
                  kv8x4_to_f16x2<kFmt>(r[2 * h + 1], a1, a3);  // d = 16(m+h) + gid + 8
                  mma_f16(ot[m + h], m0(a0), m0(a1), m1(a2), m1(a3), pa0, pa2);
                }
              }
            }
          };
          if (vh >= 16)
            pv_product(std::false_type{});
          else
            pv_product(std::true_type{});
        }
      }
    }
    if (t_flags & kSegLast) {
      // ----------------------------------------- hand the segment over
      // Each warp snapshots (m, l, o) into its slot and goes on streaming,
      // once the flush warp has read the previous segment's slots.  With two
      // slots, warps 2 and 3 do so, and warps 0 and 1 fold their partner's
      // snapshot (warp + 2) into their own state and write the result back.
      // heads h0, h1 of this thread: totals over the eight lanes of a column
      float l_h[2] = {l_part[0], l_part[1]};
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l_h[0] += __shfl_xor_sync(0xffffffffu, l_h[0], o);
        l_h[1] += __shfl_xor_sync(0xffffffffu, l_h[1], o);
      }
      const int slot = warp % kSnap;
      float* so = red_o + slot * G * kRedRow;
      const int h0 = 2 * tid4, h1 = 2 * tid4 + 1;
      // fragment rows gid and gid+8 of d-tile m hold d 16m + gid and +8
      // (bf16 and one-byte codes), or 32(m/2) + 4*gid + 2(m%2) and +1 (FP4),
      // as the PV products lay them out
      const int d_step = fp4(kFmt) ? 1 : 8;
      auto d_of = [&](int m) { return fp4(kFmt) ? 32 * (m >> 1) + 4 * gid + 2 * (m & 1) : 16 * m + gid; };
      auto write_desc = [&]() {
        const TileInfo& ti = info[stage];
        FlushDesc fd;
        fd.b = ti.b;
        fd.g = ti.g;
        fd.slot = ti.slot;
        fd.seg_base = ti.seg_base;
        fd.nseg = ti.nseg;
        fd.whole = (t_flags & kUnitWhole) ? 1 : 0;
        fd.final = (i == n_tiles - 1) ? 1 : 0;
        *desc = fd;
      };
      if (kSnap == kConsumerWarps || warp >= kSnap) {
        if (nflush > 0 && !mbar_wait(red_empty, (uint32_t)((nflush - 1) & 1), p.flags)) return;
        if (gid == 0) {
          if (h0 < G) {
            red_m[slot * G + h0] = m_run[0];
            red_l[slot * G + h0] = l_h[0];
          }
          if (h1 < G) {
            red_m[slot * G + h1] = m_run[1];
            red_l[slot * G + h1] = l_h[1];
          }
        }
        float* r0 = so + h0 * kRedRow;
        float* r1 = so + h1 * kRedRow;
#pragma unroll
        for (int m = 0; m < D / 16; ++m) {
          const int d = d_of(m);
          if (h0 < G) {
            r0[d] = ot[m][0];
            r0[d + d_step] = ot[m][2];
          }
          if (h1 < G) {
            r1[d] = ot[m][1];
            r1[d + d_step] = ot[m][3];
          }
        }
        if (kSnap == kConsumerWarps) {
          if (warp == 0 && lane == 0) write_desc();
          __syncwarp();
          if (lane == 0) mbar_arrive(red_full);
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(pair_full);
        }
      } else {
        if (!mbar_wait(pair_full, (uint32_t)(nflush & 1), p.flags)) return;
        // the partner's (m, l) of heads h0, h1 and the factors of both sides
        float M[2], sa[2], sb[2], l_new[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int h = 2 * tid4 + k;
          const float mp = h < G ? red_m[slot * G + h] : -INFINITY;
          const float lp = h < G ? red_l[slot * G + h] : 0.f;
          M[k] = fmaxf(m_run[k], mp);
          sa[k] = m_run[k] == -INFINITY ? 0.f : fast_exp2(m_run[k] - M[k]);
          sb[k] = mp == -INFINITY ? 0.f : fast_exp2(mp - M[k]);
          l_new[k] = sa[k] * l_h[k] + sb[k] * lp;
        }
        const float a_lo = sa[0], a_hi = sa[1], b_lo = sb[0], b_hi = sb[1];
        float* r0 = so + h0 * kRedRow;
        float* r1 = so + h1 * kRedRow;
#pragma unroll
        for (int m = 0; m < D / 16; ++m) {
          const int d = d_of(m);
          if (h0 < G) {
            r0[d] = ot[m][0] * a_lo + r0[d] * b_lo;
            r0[d + d_step] = ot[m][2] * a_lo + r0[d + d_step] * b_lo;
          }
          if (h1 < G) {
            r1[d] = ot[m][1] * a_hi + r1[d] * b_hi;
            r1[d + d_step] = ot[m][3] * a_hi + r1[d + d_step] * b_hi;
          }
        }
        __syncwarp();  // every lane has read the partner's (m, l)
        if (gid == 0) {
          if (h0 < G) {
            red_m[slot * G + h0] = M[0];
            red_l[slot * G + h0] = l_new[0];
          }
          if (h1 < G) {
            red_m[slot * G + h1] = M[1];
            red_l[slot * G + h1] = l_new[1];
          }
        }
        if (warp == 0 && lane == 0) write_desc();
        __syncwarp();
        if (lane == 0) mbar_arrive(red_full);
      }
      ++nflush;
    }
    // release the stage (all of this warp's reads of it are done)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
}

// --------------------------------------------------------- split reduce
// One warp per (sequence, kv head) unit whose tiles were cut across CTAs:
// out = sum_i e^{m_i - M} o_i / sum_i e^{m_i - M} l_i, lse = M + ln(...), in
// the log2 domain of the partials.  Launched as a programmatic dependent of
// the decode kernel: it may start early and waits for the decode grid's
// completion (and memory) before reading any partial.
template <int D, int G>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int u = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (u >= p.batch * p.num_kv_heads) return;
  const int b = u / p.num_kv_heads;
  const int g = u - b * p.num_kv_heads;
  const int2 info = p.unit_info[u];
  if (clamp_len(p, __ldg(p.seq_lens + b), false) == 0) return;  // written by the decode kernel
  const int n = info.y;
  if (n <= 1) return;  // whole unit: written by the decode kernel
  constexpr int GD = G * D;
  constexpr int kJ = GD / 32;  // elements of the unit's output per lane
  const int64_t mlb = (int64_t)info.x * G;
  const float* po = p.part_o + (int64_t)info.x * GD;
  // Every load of a segment (its G (m, l) pairs and this lane's kJ partial
  // outputs) is independent, so a segment costs one memory round trip and
  // consecutive segments overlap.
  float mrow[G], lrow[G], num[kJ];
#pragma unroll
  for (int r = 0; r < G; ++r) {
    mrow[r] = -INFINITY;
    lrow[r] = 0.f;
  }
#pragma unroll
  for (int j = 0; j < kJ; ++j) num[j] = 0.f;
  // pass over segments with a running (online) max per row
#pragma unroll 2
  for (int sgm = 0; sgm < n; ++sgm) {
    float2 ml[G];
    float ov[kJ];
#pragma unroll
    for (int r = 0; r < G; ++r) ml[r] = __ldcg(&p.part_ml[mlb + (int64_t)sgm * G + r]);
#pragma unroll
    for (int j = 0; j < kJ; ++j) ov[j] = __ldcg(po + (int64_t)sgm * GD + lane + 32 * j);
    float sc_old[G], sc_new[G];
#pragma unroll
    for (int r = 0; r < G; ++r) {
      const float m_new = fmaxf(mrow[r], ml[r].x);
      sc_old[r] = mrow[r] == -INFINITY ? 0.f : fast_exp2(mrow[r] - m_new);
      sc_new[r] = ml[r].x == -INFINITY ? 0.f : fast_exp2(ml[r].x - m_new);
      lrow[r] = lrow[r] * sc_old[r] + ml[r].y * sc_new[r];
      mrow[r] = m_new;
    }
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
      constexpr int kPerRow = D / 32;
      const int r = j / kPerRow;
      num[j] = num[j] * sc_old[r] + ov[j] * sc_new[r];
    }
  }
  __nv_bfloat16* ob = p.out + ((int64_t)b * p.num_q_heads + g * G) * D;
#pragma unroll
  for (int j = 0; j < kJ; ++j) {
    constexpr int kPerRow = D / 32;
    const int r = j / kPerRow;
    ob[lane + 32 * j] = __float2bfloat16(lrow[r] > 0.f ? num[j] / lrow[r] : 0.f);
  }
  if (lane == 0 && p.lse) {
#pragma unroll
    for (int r = 0; r < G; ++r)
      p.lse[(int64_t)b * p.num_q_heads + g * G + r] =
          lrow[r] > 0.f ? (mrow[r] + log2f(lrow[r])) * 0.69314718055994531f : -INFINITY;
  }
}

template <int D>
cudaError_t merge_launch(const DecodeParams& p, cudaStream_t stream) {
  const int units = p.batch * p.num_kv_heads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((units + 3) / 4);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (p.group) {
    case 1: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 2>, p);
    case 4: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 4>, p);
    default: return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D, 8>, p);
  }
}

// ------------------------------------------------------------- host side
template <int D, int kFmt, int kStages, int kSnap>
size_t decode_smem_bytes(int G) {
  return 1024 + smem_plan<D, kFmt, kStages, kSnap>(G).total;  // + alignment slack
}

template <int D, int kFmt, int kStages, int kSnap>
cudaError_t decode_prepare(int G, int* ctas_per_sm) {
  auto k = decode_kernel<D, kFmt, kStages, kSnap>;
  const size_t smem = decode_smem_bytes<D, kFmt, kStages, kSnap>(G);
  // The attribute belongs to the instantiation, which serves every group
  // size: allow the largest footprint once, not the one of this call.
  const size_t most = decode_smem_bytes<D, kFmt, kStages, kSnap>(kMaxGroup);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, k, kThreads, smem);
}

template <int D, int kFmt, int kStages, int kSnap>
cudaError_t decode_launch(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                          int num_ctas, cudaStream_t stream) {
  const size_t smem = decode_smem_bytes<D, kFmt, kStages, kSnap>(p.group);
  decode_kernel<D, kFmt, kStages, kSnap><<<num_ctas, kThreads, smem, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

// Ring depth and snapshot slots: the deepest ring that still lets two CTAs
// share an SM (228 KB of shared memory per SM, 1 KB of it reserved per CTA)
// with a slot per consumer warp, unless halving the slots buys a third stage.
constexpr size_t kSmemPerCtaFor2 = 113 * 1024;
enum class Plan { k4x4, k3x4, k3x2, k2x4 };

template <int D, int kFmt>
Plan pick_plan(int G) {
  if (decode_smem_bytes<D, kFmt, 4, 4>(G) <= kSmemPerCtaFor2) return Plan::k4x4;
  if (decode_smem_bytes<D, kFmt, 3, 4>(G) <= kSmemPerCtaFor2) return Plan::k3x4;
  if (decode_smem_bytes<D, kFmt, 3, 2>(G) <= kSmemPerCtaFor2) return Plan::k3x2;
  return Plan::k2x4;
}

template <int D, int kFmt>
cudaError_t occupancy_for(int G, int* n) {
  switch (pick_plan<D, kFmt>(G)) {
    case Plan::k4x4: return decode_prepare<D, kFmt, 4, 4>(G, n);
    case Plan::k3x4: return decode_prepare<D, kFmt, 3, 4>(G, n);
    case Plan::k3x2: return decode_prepare<D, kFmt, 3, 2>(G, n);
    default: return decode_prepare<D, kFmt, 2, 4>(G, n);
  }
}

template <int D, int kFmt>
cudaError_t run_for(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeParams& p,
                    int num_ctas, cudaStream_t stream) {
  cudaError_t e;
  switch (pick_plan<D, kFmt>(p.group)) {
    case Plan::k4x4: e = decode_launch<D, kFmt, 4, 4>(tk, tv, p, num_ctas, stream); break;
    case Plan::k3x4: e = decode_launch<D, kFmt, 3, 4>(tk, tv, p, num_ctas, stream); break;
    case Plan::k3x2: e = decode_launch<D, kFmt, 3, 2>(tk, tv, p, num_ctas, stream); break;
    default: e = decode_launch<D, kFmt, 2, 4>(tk, tv, p, num_ctas, stream); break;
  }
  if (e != cudaSuccess) return e;
  return merge_launch<D>(p, stream);
}

// Each (head_dim, format) pair is its own instantiation (and its own
// shared-memory attribute); E4M3 and INT8 share a layout, not a kernel.
cudaError_t decode_occupancy(int head_dim, int fmt, int group, int* ctas_per_sm) {
  const bool d128 = head_dim == 128;
  switch (fmt) {
    case PKV_KV_NVFP4:
      return d128 ? occupancy_for<128, PKV_KV_NVFP4>(group, ctas_per_sm)
                  : occupancy_for<64, PKV_KV_NVFP4>(group, ctas_per_sm);
    case PKV_KV_INT8:
      return d128 ? occupancy_for<128, PKV_KV_INT8>(group, ctas_per_sm)
                  : occupancy_for<64, PKV_KV_INT8>(group, ctas_per_sm);
    case PKV_KV_FP8_E4M3:
      return d128 ? occupancy_for<128, PKV_KV_FP8_E4M3>(group, ctas_per_sm)
                  : occupancy_for<64, PKV_KV_FP8_E4M3>(group, ctas_per_sm);
    default:
      return d128 ? occupancy_for<128, PKV_KV_BF16>(group, ctas_per_sm)
                  : occupancy_for<64, PKV_KV_BF16>(group, ctas_per_sm);
  }
}

cudaError_t decode_run(int head_dim, int fmt, const CUtensorMap& tk, const CUtensorMap& tv,
                       const DecodeParams& p, int num_ctas, cudaStream_t stream) {
  const bool d128 = head_dim == 128;
  switch (fmt) {
    case PKV_KV_NVFP4:
      return d128 ? run_for<128, PKV_KV_NVFP4>(tk, tv, p, num_ctas, stream)
                  : run_for<64, PKV_KV_NVFP4>(tk, tv, p, num_ctas, stream);
    case PKV_KV_INT8:
      return d128 ? run_for<128, PKV_KV_INT8>(tk, tv, p, num_ctas, stream)
                  : run_for<64, PKV_KV_INT8>(tk, tv, p, num_ctas, stream);
    case PKV_KV_FP8_E4M3:
      return d128 ? run_for<128, PKV_KV_FP8_E4M3>(tk, tv, p, num_ctas, stream)
                  : run_for<64, PKV_KV_FP8_E4M3>(tk, tv, p, num_ctas, stream);
    default:
      return d128 ? run_for<128, PKV_KV_BF16>(tk, tv, p, num_ctas, stream)
                  : run_for<64, PKV_KV_BF16>(tk, tv, p, num_ctas, stream);
  }
}

}  // namespace pkv
