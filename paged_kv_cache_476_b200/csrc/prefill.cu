// Causal prefill-chunk attention over a paged KV cache (sm_100a, tcgen05).
//
// What it computes (TensorRT-LLM concept page, "關鍵效能引數": context tokens
// are processed in parallel over the paged cache; "PagedAttention 及 KV 快取
// 管理": K/V pages found through the page table): for chunk c with n queries
// over L cached tokens, query i at position p = L - n + i attends to keys
// 0..p, out = softmax(scale * q K^T) V.
//
// Design (tensor-bound, B200-first):
//  * One CTA per (128-row Q tile, kv head, chunk).  The 128 rows pack the G
//    q heads of the kv head for 128/G consecutive query tokens (row = token *
//    G + head), so every K/V tile staged in shared memory serves the whole
//    GQA group.
//  * Warp 4 (producer) loads the Q tile once with a 3-D TMA map over
//    [token][head][d] and streams 128-key K/V tiles (one 128-token page or
//    two 64-token pages, page-table indirected, 128-byte swizzled) into a
//    two-stage mbarrier ring.
//  * Warp 5 (one elected thread) issues tcgen05.mma: S = Q K^T (M=128,
//    N=128, K=head_dim, both operands K-major from shared memory) into one
//    of two TMEM buffers, then O += P V with P (bf16) read from TMEM and V as
//    an MN-major operand.  tcgen05.commit signals completion on mbarriers.
//  * Warps 0-3 (one TMEM lane = one row per thread) run the online softmax:
//    load S from TMEM, mask the causal diagonal, keep a reference max that
//    is raised only when a row's max grows by more than 2^8 (then O is
//    rescaled in TMEM), write P to TMEM, and finally normalise O.
//  * V rows past the sequence end (or of a rejected page) are zeroed in
//    shared memory before their PV product: 0 * NaN would poison O.
//  * Every wait is bounded; TMEM is freed on every exit path.
#include "common.cuh"
#include "kernels.h"

namespace pkv {

namespace pf {

constexpr int kRows = 128;     // M of the Q tile
constexpr int kKeys = 128;     // N of the S tile (keys per KV tile)
constexpr int kStages = 2;     // K/V ring depth
constexpr int kThreads = 192;  // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP = 384;

struct Params {
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

// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, M x N, operand majors.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major) {
  return (1u << 4)                         // D format f32
         | (1u << 7)                       // A bf16
         | (1u << 10)                      // B bf16
         | ((uint32_t)b_mn_major << 16)    // B major: 0 K, 1 MN
         | ((uint32_t)(N >> 3) << 17)      // N / 8
         | ((uint32_t)(M >> 4) << 24);     // M / 16
}

template <int D>
struct Smem {
  static constexpr int kHalves = D / 64;          // 128-byte column boxes per row
  static constexpr int kQB = kRows * D * 2;       // Q tile
  static constexpr int kTileB = kKeys * D * 2;    // K (or V) tile
  static constexpr int kHalfB = kKeys * 128;      // one 64-column half of a K/V tile
  static constexpr int kStageB = 2 * kTileB;
  static constexpr int kBytes = kQB + kStages * kStageB;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const Params p) {
  using Sm = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = smem;
  uint8_t* skv = smem + Sm::kQB;  // stage s: K at s*kStageB, V at +kTileB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sm::kBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;             // [kStages]
  uint64_t* kv_empty = kv_full + kStages;   // [kStages]
  uint64_t* s_full = kv_empty + kStages;    // [2]
  uint64_t* s_free = s_full + 2;            // [2]
  uint64_t* p_full = s_free + 2;
  uint64_t* o_bar = p_full + 1;
  uint64_t* done_bar = o_bar + 1;
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(done_bar + 1);
  int32_t* stage_bad = reinterpret_cast<int32_t*>(tmem_base_smem + 1);  // [kStages] bit/sub-block
  int32_t* s_abort = stage_bad + kStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.group;
  const int TQ = kRows / G;  // query tokens per tile
  const int chunk = blockIdx.z;
  const int g = blockIdx.y;
  const int qt0 = blockIdx.x * TQ;

  const int32_t q_begin = __ldg(p.cu_q + chunk);
  const int32_t n = __ldg(p.cu_q + chunk + 1) - q_begin;
  int32_t L = __ldg(p.seq_lens + chunk);
  if (n <= 0 || qt0 >= n) return;  // uniform across the CTA
  const int32_t cap = p.max_pages * p.page_size;
  if (L > cap || n > L) {
    if (threadIdx.x == 0) flag_error(p.flags, PKV_FLAG_BAD_LENGTH);
    if (n > cap || L < n) return;  // nothing meaningful to compute
    L = min(L, cap);
  }
  const int tq_end = min(qt0 + TQ, n);                 // exclusive token bound of this tile
  const int32_t p_max = L - n + tq_end - 1;            // largest query position
  const int32_t p_min = L - n + qt0;                   // smallest query position
  const int n_kv = (p_max + kKeys) / kKeys;            // KV tiles to visit

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(o_bar, 1);
    mbar_init(done_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(tmem_base_smem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      mbar_arrive_expect_tx(q_full, (uint32_t)Sm::kQB);
#pragma unroll
      for (int h = 0; h < Sm::kHalves; ++h)
        tma_load_3d(sq + h * (kRows * 128), &tmap_q, h * 64, g * G, q_begin + qt0, q_full);
    }
    const uint64_t pol = policy_evict_first();
    (void)pol;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j % kStages;
      if (j >= kStages) {
        if (!mbar_wait(&kv_empty[st], (uint32_t)((j / kStages - 1) & 1), p.flags)) {
          *s_abort = 1;
          break;
        }
      }
      if (lane == 0) {
        uint8_t* kd = skv + st * Sm::kStageB;
        uint8_t* vd = kd + Sm::kTileB;
        int bad = 0;
        uint32_t bytes = 0;
        int32_t ys[2] = {0, 0};
        bool live[2] = {false, false};
        for (int sb = 0; sb < 2; ++sb) {
          const int32_t key0 = j * kKeys + sb * 64;
          if (key0 >= L) continue;
          const int32_t pj = key0 / p.page_size;
          int32_t pid = __ldg(p.page_table + (int64_t)chunk * p.max_pages + pj);
          if (pid < 0 || pid >= p.num_pages) {
            flag_error(p.flags, PKV_FLAG_BAD_PAGE);
            bad |= 1 << sb;
            continue;
          }
          ys[sb] = (int32_t)(((int64_t)pid * p.num_kv_heads + g) * p.page_size +
                             key0 % p.page_size);
          live[sb] = true;
          bytes += 2u * Sm::kHalves * 64u * 128u;
        }
        stage_bad[st] = bad;
        mbar_arrive_expect_tx(&kv_full[st], bytes);
        for (int sb = 0; sb < 2; ++sb) {
          if (!live[sb]) continue;
#pragma unroll
          for (int h = 0; h < Sm::kHalves; ++h) {
            tma_load_2d(kd + h * Sm::kHalfB + sb * 64 * 128, &tmap_k, h * 64, ys[sb],
                        &kv_full[st], pol);
            tma_load_2d(vd + h * Sm::kHalfB + sb * 64 * 128, &tmap_v, h * 64, ys[sb],
                        &kv_full[st], pol);
          }
        }
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    const uint32_t id_s = idesc_bf16(kRows, kKeys, 0);
    const uint32_t id_o = idesc_bf16(kRows, D, 1);
    const uint32_t q_addr = smem_u32(sq);
    bool ok = mbar_wait(q_full, 0, p.flags);
    auto issue_pv = [&](int i) -> bool {
      const int st = i % kStages;
      if (!mbar_wait(p_full, (uint32_t)(i & 1), p.flags)) return false;
      tc_fence_after();
      // zero V rows that must not contribute (past the end, or a rejected page)
      const int32_t key0 = i * kKeys;
      const int bad = stage_bad[st];
      int zlo = kKeys;  // first row to zero (tail)
      if (key0 + kKeys > L) zlo = max(0, L - key0);
      if (zlo < kKeys || bad) {
        uint8_t* vd = skv + st * Sm::kStageB + Sm::kTileB;
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
      if (lane == 0) {
        const uint32_t v_addr = smem_u32(skv + st * Sm::kStageB + Sm::kTileB);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          // B = V [keys x d], MN-major: 8-key groups 1024 B apart (SBO), the
          // 64-column halves kHalfB apart (LBO).
          const uint64_t bd = sdesc(v_addr + kk * 2048, Sm::kHalfB, 1024);
          mma_ts(tmem + kColO, tmem + kColP + kk * 8, bd, id_o, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(o_bar);
        tc_commit(&kv_empty[st]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < n_kv && ok; ++j) {
      const int st = j % kStages;
      const int sb = j & 1;
      if (!mbar_wait(&kv_full[st], (uint32_t)((j / kStages) & 1), p.flags)) { ok = false; break; }
      if (j >= 2 && !mbar_wait(&s_free[sb], (uint32_t)((j / 2 - 1) & 1), p.flags)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t k_addr = smem_u32(skv + st * Sm::kStageB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // A = Q, B = K, both K-major: 16-element K steps advance 32 B inside
          // a 128-byte swizzled row; the second 64 columns live kHalfB away.
          const int h = kk >> 2, w = kk & 3;
          const uint64_t ad = sdesc(q_addr + h * (kRows * 128) + w * 32, 16, 1024);
          const uint64_t bd = sdesc(k_addr + h * Sm::kHalfB + w * 32, 16, 1024);
          mma_ss(tmem + (sb ? kColS1 : kColS0), ad, bd, id_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
      }
      __syncwarp();
      if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok && n_kv > 0) ok = issue_pv(n_kv - 1);
    if (!ok) *s_abort = 1;
    // every MMA this thread issued must finish before TMEM is released
    if (lane == 0) tc_commit(done_bar);
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int r = threadIdx.x;  // row = TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int t_local = qt0 + r / G;
    const bool row_ok = t_local < n;
    const int32_t pos = row_ok ? L - n + t_local : p_max;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      const int st = j % kStages;
      if (!mbar_wait(&s_full[sb], (uint32_t)((j / 2) & 1), p.flags)) { ok = false; break; }
      if (!mbar_wait(&kv_full[st], (uint32_t)((j / kStages) & 1), p.flags)) { ok = false; break; }
      const int bad = stage_bad[st];
      tc_fence_after();
      float s[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys; c += 32)
        tmem_ld32(tmem + lane_base + (sb ? kColS1 : kColS0) + c, s + c);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      // mask: causal diagonal (which also covers keys past the end) and
      // sub-blocks of a rejected page
      const int32_t key0 = j * kKeys;
      const bool diag = key0 + kKeys - 1 > p_min;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; ++c) {
        const int32_t key = key0 + c;
        const bool keep = (!diag || key <= pos) && !((bad >> (c >> 6)) & 1);
        s[c] = keep ? s[c] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[c]);
      }
      const bool need = mt > m_ref + 8.f;  // also true on the first visible tile
      // PV of the previous tile must be done before P is overwritten or O rescaled
      if (j >= 1 && !mbar_wait(o_bar, (uint32_t)((j - 1) & 1), p.flags)) { ok = false; break; }
      tc_fence_after();
      const float m_new = need ? mt : m_ref;
      if (j >= 1 && __any_sync(0xffffffffu, need)) {
        const float alpha = need ? fast_exp2(m_ref - m_new) : 1.f;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + kColO + c, o);
          tmem_wait_ld();
          uint32_t u[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(o[i] * alpha);
          tmem_st16(tmem + lane_base + kColO + c, u);
          tmem_st16(tmem + lane_base + kColO + c + 16, u + 16);
        }
        l *= alpha;
      }
      m_ref = m_new;
      // a row with no visible key yet keeps m_ref = -inf: its p must be 0
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      uint32_t pk[kKeys / 2];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kKeys; c += 2) {
        const float p0 = fast_exp2(s[c] - m_use);
        const float p1 = fast_exp2(s[c + 1] - m_use);
        rs += p0 + p1;
        pk[c / 2] = pack_bf16(p0, p1);
      }
      l += rs;
#pragma unroll
      for (int c = 0; c < kKeys / 2; c += 16) tmem_st16(tmem + lane_base + kColP + c, pk + c);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // -------------------------------------------------------- epilogue
    if (ok && n_kv > 0 && mbar_wait(o_bar, (uint32_t)((n_kv - 1) & 1), p.flags)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t qrow = (int64_t)q_begin + t_local;
      const int h = g * G + (r % G);
      __nv_bfloat16* dst = p.out + (qrow * p.num_q_heads + h) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + kColO + c, o);
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

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kProducerWarp) {
    // no bulk copy may still be landing in shared memory when the CTA exits
    for (int j = max(0, n_kv - kStages); j < n_kv; ++j)
      mbar_wait(&kv_full[j % kStages], (uint32_t)((j / kStages) & 1), p.flags);
  }
  if (warp == kMmaWarp) {
    mbar_wait(done_bar, 0, p.flags);
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
size_t smem_bytes() {
  return 1024 + Smem<D>::kBytes + 16 * sizeof(uint64_t) + 16 * sizeof(int32_t);
}

template <int D>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const Params& p, int q_tiles, cudaStream_t stream) {
  const size_t smem = smem_bytes<D>();
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(q_tiles, p.num_kv_heads, p.num_chunks);
  prefill_kernel<D><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
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
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PKV_ERR_SHAPE;
  if (num_chunks == 0 || total_q == 0 || max_q_len == 0) return PKV_OK;
  if (!q || !cu_q_lens || !page_table || !seq_lens || !out) return PKV_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
    return PKV_ERR_ALIGN;
  if (cache->kv_dtype != PKV_KV_BF16) return PKV_ERR_UNSUPPORTED;
  const int D = cache->head_dim;
  CUtensorMap tq, tk, tv;
  if ((st = encode_q_map(&tq, q, total_q, num_q_heads, D, gqa_group))) return st;
  const int64_t rows = (int64_t)cache->num_pages * cache->num_kv_heads * cache->page_size;
  if ((st = encode_pool_map(&tk, cache->k_pool, false, rows, D, 64, 64))) return st;
  if ((st = encode_pool_map(&tv, cache->v_pool, false, rows, D, 64, 64))) return st;
  pf::Params p;
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
  const int tq_tokens = pf::kRows / gqa_group;
  const int q_tiles = (max_q_len + tq_tokens - 1) / tq_tokens;
  cudaError_t e = D == 128 ? pf::launch<128>(tq, tk, tv, p, q_tiles, stream)
                           : pf::launch<64>(tq, tk, tv, p, q_tiles, stream);
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
