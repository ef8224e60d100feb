/*
 * CPU oracle for attention over a paged KV cache.  TEST INFRASTRUCTURE ONLY:
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * load this file's library.  It shares no code with the CUDA path.
 *
 * Every function is the plain definition, written for a reader to check by
 * eye: no blocking, no fusion, no reordering.  Floating point is fp64, except
 * the FP8 quantisation quotient, which is an fp32 IEEE division because the
 * stored code is decided in the precision the kernel uses (an fp32 scale and
 * an fp32 quotient), then rounded by the exact E4M3 encoder below.
 *
 * Sources (the pages on TensorRT-LLM):
 *  - TensorRT-LLM concept page (compassingai.com), "關鍵機制 / PagedAttention
 *    及 KV 快取管理": each sequence's KV cache is cut into fixed-size pages
 *    (64 or 128 tokens); a page table maps logical token positions to
 *    physical pages; pages are added as a sequence grows.
 *  - same page, "技術原理 / 編譯期圖最佳化": page-table lookup nodes map the
 *    logical token position of every KV read and write to its physical page.
 *  - same page, "執行時執行模型": in each forward pass the attention operator
 *    reads and updates the KV pages.
 *  - same page, "關鍵效能引數": context (prefill) tokens are processed in
 *    parallel over the paged cache.
 *  - yololab.net optimisation guide, "FP8 與極致量化": FP8 halves the bytes.
 * The attention itself is textbook softmax(Q K^T * scale) V over the tokens
 * gathered through the page table into a contiguous buffer.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *  - pool layout [page][kv_head][slot][head_dim], separate K and V pools;
 *  - page table int32 [seq][max_pages_per_seq]; entry j covers tokens
 *    [j*P, (j+1)*P); entries past the last needed page are ignored;
 *  - q head h reads kv head h / (Hq/Hkv);
 *  - softmax scale multiplies Q.K before the max; natural exp/log; lse is
 *    the natural-log sum-exp of the scaled scores;
 *  - prefill chunk query i of a chunk with n queries over L tokens sits at
 *    position L-n+i and sees keys 0..L-n+i inclusive;
 *  - FP8: E4M3 (bias 7, no infinities, 0x7F/0xFF NaN, max 448) with one fp32
 *    scale per (page, kv head) for K and one for V; stored code =
 *    e4m3_rne_satfinite(fp32(x) / scale); value = decode(code) * scale;
 *  - INT8 (the concept page's INT8 KV-cache quantisation, "關鍵機制"
 *    quantisation bullet): the same per-(page, kv head) scales; stored code =
 *    round-half-even of the fp32 quotient clamped to [-127, 127] (-128 never
 *    stored), NaN -> 0; value = code * scale;
 *  - NVFP4 (the pages: FP4 quantisation needs Blackwell; codec only so far):
 *    E2M1 codes, an E4M3 scale per 16 head_dim values of a row, and the same
 *    per-(page, kv head) fp32 scale; see the NVFP4 section below;
 *  - a sequence of length 0 yields out = 0 and lse = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_PAGE (-2)
#define ORC_ERR_LEN (-3)
#define ORC_ERR_NOMEM (-4)

#define KV_BF16 0
#define KV_E4M3 1
#define KV_INT8 2
#define KV_NVFP4 3

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads of the OpenMP loops from now on (n >= 1). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------ bf16 */
/* A bf16 value is the upper half of an IEEE binary32; widening is exact. */
static double bf16_value(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static float bf16_to_f32(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* ------------------------------------------------------------------ E4M3 */
/*
 * E4M3 (the "fn" variant used for FP8 KV): 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits.
 *   exponent field 0:      value = m/8 * 2^-6  = m * 2^-9     (subnormal)
 *   exponent field 1..15:  value = (1 + m/8) * 2^(e-7)
 *   e = 15, m = 7:         NaN (no infinities); largest finite 448.
 */
double oracle_e4m3_decode(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexp((double)m, -9);
  else
    mag = ldexp(8.0 + m, e - 10);
  return sign ? -mag : mag;
}

/*
 * Round an fp32 value to the nearest E4M3 value, ties to an even mantissa
 * code, saturating anything that rounds above 448 (including +-inf) to +-448.
 * The sign is kept for zero and for values that round to zero.  NaN maps to
 * the NaN code with the input's sign.
 */
uint8_t oracle_e4m3_encode(float y) {
  uint8_t sign = signbit(y) ? 0x80 : 0x00;
  double a = fabs((double)y);
  if (isnan(y)) return (uint8_t)(sign | 0x7F);
  if (isinf(y) || a >= 448.0) return (uint8_t)(sign | 0x7E);
  /* The spacing of E4M3 values around a: 2^-9 below the smallest normal
   * 2^-6, else 2^(E-3) where 2^E <= a < 2^(E+1). */
  int E;
  double quantum;
  if (a < ldexp(1.0, -6)) {
    quantum = ldexp(1.0, -9);
  } else {
    frexp(a, &E); /* a = f * 2^E with f in [0.5, 1) */
    E -= 1;       /* now 2^E <= a < 2^(E+1) */
    quantum = ldexp(1.0, E - 3);
  }
  double steps = a / quantum;          /* exact: quantum is a power of two */
  double n = nearbyint(steps);         /* default rounding: nearest, ties to even */
  double v = n * quantum;              /* the rounded magnitude */
  if (v > 448.0) return (uint8_t)(sign | 0x7E);
  if (v < ldexp(1.0, -6)) {            /* subnormal (or zero): code = v / 2^-9 */
    int k = (int)(v / ldexp(1.0, -9));
    return (uint8_t)(sign | k);
  }
  int Ev;
  frexp(v, &Ev);
  Ev -= 1;                             /* 2^Ev <= v < 2^(Ev+1) */
  int mant = (int)((v / ldexp(1.0, Ev) - 1.0) * 8.0); /* exact, 0..7 */
  int efield = Ev + 7;
  return (uint8_t)(sign | (efield << 3) | mant);
}

/* The fp32 IEEE quotient the stored code is decided from. */
float oracle_fp8_quotient(uint16_t x_bits, float scale) {
  volatile float x = bf16_to_f32(x_bits);
  volatile float q = x / scale;
  return q;
}

uint8_t oracle_fp8_quantize(uint16_t x_bits, float scale) {
  return oracle_e4m3_encode(oracle_fp8_quotient(x_bits, scale));
}

/* ------------------------------------------------------------------ INT8 */
/*
 * Symmetric INT8: the nearest integer to y, ties to even, clamped to
 * [-127, 127] (so -128 is never produced and +-inf give +-127); NaN gives 0.
 */
int8_t oracle_int8_encode(float y) {
  if (isnan(y)) return 0;
  double a = (double)y;
  if (a > 127.0) a = 127.0;
  if (a < -127.0) a = -127.0;
  return (int8_t)nearbyint(a); /* default rounding: nearest, ties to even */
}

int8_t oracle_int8_quantize(uint16_t x_bits, float scale) {
  return oracle_int8_encode(oracle_fp8_quotient(x_bits, scale));
}

void oracle_int8_quantize_array(const uint16_t* x_bits, const float* scale, int8_t* codes,
                                int64_t n) {
  for (int64_t i = 0; i < n; ++i) codes[i] = oracle_int8_quantize(x_bits[i], scale[i]);
}

/* ----------------------------------------------------------------- NVFP4 */
/*
 * FP4 pools (the pages say only that FP4 quantisation needs Blackwell; the
 * layout below is this library's reading): E2M1 element codes; the 16
 * consecutive head_dim values of one (token, kv head) row share an E4M3
 * block scale; the per-(page, kv head) fp32 scale of the other one-byte
 * formats multiplies both.
 *
 * E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; no infinities, no NaN.
 *   exponent field 0:      value = m * 0.5                 (0, 0.5)
 *   exponent field 1..3:   value = (1 + m/2) * 2^(e-1)     (1 ... 6)
 */
double oracle_e2m1_decode(uint8_t code) {
  int sign = (code >> 3) & 1;
  int e = (code >> 1) & 3;
  int m = code & 1;
  double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -mag : mag;
}

/*
 * Nearest E2M1 value, ties to an even mantissa code; anything at or above 6
 * (+-inf included) saturates to +-6.  The sign is kept for zero and for
 * values that round to zero; NaN gives +0 (E2M1 has no NaN).
 */
uint8_t oracle_e2m1_encode(float y) {
  static const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  if (isnan(y)) return 0;
  uint8_t sign = signbit(y) ? 8 : 0;
  double a = fabs((double)y);
  if (a >= 6.0) return (uint8_t)(sign | 7);
  /* spacing of the grid around a: 0.5 on [0, 2), 1 on [2, 4), 2 on [4, 6] */
  double quantum = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
  /* nearest multiple, ties to the even multiple: on every stretch the even
   * multiples are exactly the even codes */
  double v = nearbyint(a / quantum) * quantum;
  for (int c = 0; c < 8; ++c)
    if (mags[c] == v) return (uint8_t)(sign | c);
  return (uint8_t)(sign | 7); /* not reached: v is on the grid */
}

/*
 * One row of n values (n a multiple of 16) of a (page, kv head) whose fp32
 * scale is s, block by block:
 *   amax   = max |x| over the block's 16 values (NaN ignored)
 *   sb     = e4m3_rne_satfinite(fp32(amax / fp32(6 * s)))     block scale code
 *   d      = fp32(decode(sb) * s)                              the block's unit
 *   code_i = e2m1_encode(d > 0 ? fp32(x_i / d) : 0)
 * so that value_i = e2m1(code_i) * decode(sb) * s.  Two codes per byte, the
 * even element in the low nibble; one block-scale byte per 16 values.
 */
void oracle_nvfp4_quantize_row(const uint16_t* x_bits, int64_t n, float s, uint8_t* packed,
                               uint8_t* block_scales) {
  for (int64_t b = 0; b < n / 16; ++b) {
    float amax = 0.f;
    for (int i = 0; i < 16; ++i) {
      float x = bf16_to_f32(x_bits[b * 16 + i]);
      if (!isnan(x) && fabsf(x) > amax) amax = fabsf(x);
    }
    volatile float six_s = 6.0f * s;
    volatile float ratio = amax / six_s;
    uint8_t sb = oracle_e4m3_encode(ratio);
    volatile float d = (float)oracle_e4m3_decode(sb) * s;
    block_scales[b] = sb;
    for (int i = 0; i < 16; i += 2) {
      uint8_t c[2];
      for (int k = 0; k < 2; ++k) {
        volatile float x = bf16_to_f32(x_bits[b * 16 + i + k]);
        volatile float y = d > 0.f ? x / d : 0.f;
        c[k] = oracle_e2m1_encode(y);
      }
      packed[(b * 16 + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));
    }
  }
}

/* The stored value of element i of a row quantised as above, in fp64 (exact). */
double oracle_nvfp4_value(const uint8_t* packed, const uint8_t* block_scales, float s,
                          int64_t i) {
  uint8_t byte = packed[i / 2];
  uint8_t code = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
  return oracle_e2m1_decode(code) * oracle_e4m3_decode(block_scales[i / 16]) * (double)s;
}

void oracle_e2m1_encode_array(const float* y, uint8_t* codes, int64_t n) {
  for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e2m1_encode(y[i]);
}

/* Array helpers for exhaustive codec checks. */
void oracle_e4m3_encode_array(const float* y, uint8_t* codes, int64_t n) {
  for (int64_t i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode(y[i]);
}

void oracle_e4m3_decode_array(const uint8_t* codes, double* v, int64_t n) {
  for (int64_t i = 0; i < n; ++i) v[i] = oracle_e4m3_decode(codes[i]);
}

void oracle_fp8_quantize_array(const uint16_t* x_bits, const float* scale, uint8_t* codes,
                               int64_t n) {
  for (int64_t i = 0; i < n; ++i) codes[i] = oracle_fp8_quantize(x_bits[i], scale[i]);
}

/* ------------------------------------------------------------- the cache */
typedef struct {
  uint8_t* k_pool;
  uint8_t* v_pool;
  const float* k_scale; /* [num_pages][num_kv_heads], E4M3 and INT8 only */
  const float* v_scale;
  int kv_dtype;
  int num_pages;
  int page_size;
  int num_kv_heads;
  int head_dim;
} cache_t;

static int elem_bytes(int kv_dtype) { return kv_dtype == KV_BF16 ? 2 : 1; }

/* Index of the pool row (page, kv head, slot). */
static int64_t row_index(const cache_t* c, int64_t page, int g, int slot) {
  return (page * c->num_kv_heads + g) * (int64_t)c->page_size + slot;
}

/*
 * FP4 pools hold two regions, rows in the same [page][kv head][slot] order:
 * the codes (head_dim / 2 bytes a row, two per byte, the even element in the
 * low nibble), then the E4M3 block scales (head_dim / 16 bytes a row).
 */
static int64_t nvfp4_codes_bytes(const cache_t* c) {
  return (int64_t)c->num_pages * c->num_kv_heads * c->page_size * (c->head_dim / 2);
}

/* Byte offset of element (page, kv head, slot, d) in a pool: for FP4 pools,
 * the byte holding its code. */
static int64_t pool_offset(const cache_t* c, int64_t page, int g, int slot, int d) {
  if (c->kv_dtype == KV_NVFP4) return row_index(c, page, g, slot) * (c->head_dim / 2) + d / 2;
  return (row_index(c, page, g, slot) * c->head_dim + d) * elem_bytes(c->kv_dtype);
}

/* Byte offset of the block scale of element d of row (page, kv head, slot). */
static int64_t nvfp4_scale_offset(const cache_t* c, int64_t page, int g, int slot, int d) {
  return nvfp4_codes_bytes(c) + row_index(c, page, g, slot) * (c->head_dim / 16) + d / 16;
}

/* Physical page holding logical token t of a sequence (page table lookup). */
static int lookup_page(const cache_t* c, const int32_t* table_row, int max_pages, int64_t t,
                       int64_t* page) {
  int64_t j = t / c->page_size;
  if (j >= max_pages) return ORC_ERR_LEN;
  int32_t p = table_row[j];
  if (p < 0 || p >= c->num_pages) return ORC_ERR_PAGE;
  *page = p;
  return ORC_OK;
}

/* The value of one stored element, in fp64. */
static double stored_value(const cache_t* c, const uint8_t* pool, const float* scale,
                           int64_t page, int g, int slot, int d) {
  int64_t off = pool_offset(c, page, g, slot, d);
  if (c->kv_dtype == KV_E4M3)
    return oracle_e4m3_decode(pool[off]) * (double)scale[page * c->num_kv_heads + g];
  if (c->kv_dtype == KV_INT8)
    return (double)(int8_t)pool[off] * (double)scale[page * c->num_kv_heads + g];
  if (c->kv_dtype == KV_NVFP4) {
    uint8_t code = (d & 1) ? (uint8_t)(pool[off] >> 4) : (uint8_t)(pool[off] & 0xF);
    uint8_t sb = pool[nvfp4_scale_offset(c, page, g, slot, d)];
    return oracle_e2m1_decode(code) * oracle_e4m3_decode(sb) *
           (double)scale[page * c->num_kv_heads + g];
  }
  uint16_t bits;
  memcpy(&bits, pool + off, 2);
  return bf16_value(bits);
}

static int check_cache(const cache_t* c) {
  if (!c->k_pool || !c->v_pool) return ORC_ERR_ARG;
  if (c->kv_dtype != KV_BF16 && c->kv_dtype != KV_E4M3 && c->kv_dtype != KV_INT8 &&
      c->kv_dtype != KV_NVFP4)
    return ORC_ERR_ARG;
  if (c->kv_dtype == KV_NVFP4 && c->head_dim % 16) return ORC_ERR_ARG;
  if (c->kv_dtype != KV_BF16 && (!c->k_scale || !c->v_scale)) return ORC_ERR_ARG;
  if (c->num_pages < 0 || c->page_size <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0)
    return ORC_ERR_ARG;
  return ORC_OK;
}

/* ---------------------------------------------------------------- append */
/*
 * Paged KV store.  New token j of sequence b sits at logical position
 * pos = seq_lens_before[b] + j; its page is page_table[b][pos / P] and its
 * slot pos % P.  bf16 stores the input bits; E4M3 and INT8 store the
 * quantised code; FP4 stores the row's codes and block scales.
 * k_new/v_new: bf16 bits [total_new][num_kv_heads][head_dim], ordered by
 * sequence through cu_new [batch+1].
 */
int oracle_append(uint8_t* k_pool, uint8_t* v_pool, const float* k_scale, const float* v_scale,
                  int kv_dtype, int num_pages, int page_size, int num_kv_heads, int head_dim,
                  const int32_t* page_table, int max_pages_per_seq,
                  const int32_t* seq_lens_before, const int32_t* cu_new, int batch,
                  const uint16_t* k_new, const uint16_t* v_new) {
  cache_t c = {k_pool, v_pool, k_scale, v_scale, kv_dtype, num_pages, page_size, num_kv_heads,
               head_dim};
  int st = check_cache(&c);
  if (st) return st;
  if (batch < 0 || (batch > 0 && (!page_table || !seq_lens_before || !cu_new))) return ORC_ERR_ARG;
  for (int b = 0; b < batch; ++b) {
    const int32_t* row = page_table + (int64_t)b * max_pages_per_seq;
    for (int64_t j = cu_new[b]; j < cu_new[b + 1]; ++j) {
      int64_t pos = (int64_t)seq_lens_before[b] + (j - cu_new[b]);
      int64_t page;
      st = lookup_page(&c, row, max_pages_per_seq, pos, &page);
      if (st) return st;
      int slot = (int)(pos % page_size);
      for (int g = 0; g < num_kv_heads; ++g) {
        if (kv_dtype == KV_NVFP4) { /* the whole row: its blocks share scales */
          int64_t src = (j * num_kv_heads + g) * (int64_t)head_dim;
          int64_t r = row_index(&c, page, g, slot);
          float ks = k_scale[page * num_kv_heads + g];
          float vs = v_scale[page * num_kv_heads + g];
          oracle_nvfp4_quantize_row(k_new + src, head_dim, ks, k_pool + r * (head_dim / 2),
                                    k_pool + nvfp4_codes_bytes(&c) + r * (head_dim / 16));
          oracle_nvfp4_quantize_row(v_new + src, head_dim, vs, v_pool + r * (head_dim / 2),
                                    v_pool + nvfp4_codes_bytes(&c) + r * (head_dim / 16));
          continue;
        }
        for (int d = 0; d < head_dim; ++d) {
          int64_t src = (j * num_kv_heads + g) * (int64_t)head_dim + d;
          int64_t off = pool_offset(&c, page, g, slot, d);
          if (kv_dtype == KV_E4M3) {
            float ks = k_scale[page * num_kv_heads + g];
            float vs = v_scale[page * num_kv_heads + g];
            k_pool[off] = oracle_fp8_quantize(k_new[src], ks);
            v_pool[off] = oracle_fp8_quantize(v_new[src], vs);
          } else if (kv_dtype == KV_INT8) {
            float ks = k_scale[page * num_kv_heads + g];
            float vs = v_scale[page * num_kv_heads + g];
            k_pool[off] = (uint8_t)oracle_int8_quantize(k_new[src], ks);
            v_pool[off] = (uint8_t)oracle_int8_quantize(v_new[src], vs);
          } else {
            memcpy(k_pool + off, &k_new[src], 2);
            memcpy(v_pool + off, &v_new[src], 2);
          }
        }
      }
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------- attention */
/*
 * Gather tokens [0, n) of kv head g of one sequence into contiguous fp64
 * buffers K[n][D], V[n][D] through the page table.
 */
static int gather(const cache_t* c, const int32_t* row, int max_pages, int g, int64_t n,
                  double* K, double* V) {
  for (int64_t t = 0; t < n; ++t) {
    int64_t page;
    int st = lookup_page(c, row, max_pages, t, &page);
    if (st) return st;
    int slot = (int)(t % c->page_size);
    for (int d = 0; d < c->head_dim; ++d) {
      K[t * c->head_dim + d] = stored_value(c, c->k_pool, c->k_scale, page, g, slot, d);
      V[t * c->head_dim + d] = stored_value(c, c->v_pool, c->v_scale, page, g, slot, d);
    }
  }
  return ORC_OK;
}

/*
 * Textbook attention of one query row over keys [0, n):
 *   s_t = scale * sum_d q[d] K[t][d],  m = max_t s_t,
 *   o   = sum_t exp(s_t - m) V[t] / sum_t exp(s_t - m),
 *   lse = m + log(sum_t exp(s_t - m)).
 * s is scratch of length >= n.
 */
static void attend_row(const double* q, const double* K, const double* V, int64_t n, int D,
                       double scale, double* s, double* o, double* lse) {
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (n <= 0) {
    *lse = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int64_t t = 0; t < n; ++t) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += q[d] * K[t * D + d];
    s[t] = scale * dot;
    if (s[t] > m) m = s[t];
  }
  double den = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    double e = exp(s[t] - m);
    den += e;
    for (int d = 0; d < D; ++d) o[d] += e * V[t * D + d];
  }
  for (int d = 0; d < D; ++d) o[d] /= den;
  *lse = m + log(den);
}

/*
 * Decode attention: one query token per sequence.
 * q: bf16 bits [batch][num_q_heads][head_dim]; seq_lens: tokens per sequence
 * after the append.  out: fp64 [batch][num_q_heads][head_dim]; lse: fp64
 * [batch][num_q_heads] (may be NULL).  seq_ids (optional, n_ids entries)
 * restricts the work to those sequences; other rows of out/lse are untouched.
 */
int oracle_decode(const uint8_t* k_pool, const uint8_t* v_pool, const float* k_scale,
                  const float* v_scale, int kv_dtype, int num_pages, int page_size,
                  int num_kv_heads, int head_dim, const uint16_t* q, int num_q_heads,
                  const int32_t* page_table, int max_pages_per_seq, const int32_t* seq_lens,
                  int batch, double softmax_scale, const int32_t* seq_ids, int n_ids,
                  double* out, double* lse) {
  cache_t c = {(uint8_t*)k_pool, (uint8_t*)v_pool, k_scale, v_scale, kv_dtype, num_pages,
               page_size, num_kv_heads, head_dim};
  int st = check_cache(&c);
  if (st) return st;
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads) return ORC_ERR_ARG;
  const int G = num_q_heads / num_kv_heads;
  const int D = head_dim;
  const int nb = seq_ids ? n_ids : batch;
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < (int64_t)nb * num_kv_heads; ++u) {
    int b = seq_ids ? seq_ids[u / num_kv_heads] : (int)(u / num_kv_heads);
    int g = (int)(u % num_kv_heads);
    int64_t n = seq_lens[b];
    if (b < 0 || b >= batch || n < 0) {
#pragma omp atomic write
      err = ORC_ERR_ARG;
      continue;
    }
    double* K = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
    double* V = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
    double* s = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* qd = malloc(sizeof(double) * D);
    double lse_h;
    if (!K || !V || !s || !qd) {
#pragma omp atomic write
      err = ORC_ERR_NOMEM;
    } else {
      int gs = gather(&c, page_table + (int64_t)b * max_pages_per_seq, max_pages_per_seq, g, n,
                      K, V);
      if (gs) {
#pragma omp atomic write
        err = gs;
      } else {
        for (int h = g * G; h < (g + 1) * G; ++h) {
          for (int d = 0; d < D; ++d)
            qd[d] = bf16_value(q[((int64_t)b * num_q_heads + h) * D + d]);
          attend_row(qd, K, V, n, D, softmax_scale, s,
                     out + ((int64_t)b * num_q_heads + h) * D, &lse_h);
          if (lse) lse[(int64_t)b * num_q_heads + h] = lse_h;
        }
      }
    }
    free(K);
    free(V);
    free(s);
    free(qd);
  }
  return err;
}

/*
 * Causal prefill-chunk attention.  Chunk c owns queries [cu_q[c], cu_q[c+1])
 * of the packed q (bf16 bits [T_q][num_q_heads][head_dim]) and has
 * seq_lens[c] tokens in the cache after the append.  Query i of the chunk
 * (n queries) sits at position p = seq_lens[c] - n + i and attends to keys
 * 0..p inclusive.  out: fp64 [T_q][num_q_heads][head_dim]; lse: [T_q][Hq].
 */
int oracle_prefill_chunk(const uint8_t* k_pool, const uint8_t* v_pool, const float* k_scale,
                         const float* v_scale, int kv_dtype, int num_pages, int page_size,
                         int num_kv_heads, int head_dim, const uint16_t* q, int num_q_heads,
                         const int32_t* cu_q, const int32_t* page_table, int max_pages_per_seq,
                         const int32_t* seq_lens, int num_chunks, double softmax_scale,
                         double* out, double* lse) {
  cache_t c = {(uint8_t*)k_pool, (uint8_t*)v_pool, k_scale, v_scale, kv_dtype, num_pages,
               page_size, num_kv_heads, head_dim};
  int st = check_cache(&c);
  if (st) return st;
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads) return ORC_ERR_ARG;
  const int G = num_q_heads / num_kv_heads;
  const int D = head_dim;
  for (int ch = 0; ch < num_chunks; ++ch) {
    int64_t nq = (int64_t)cu_q[ch + 1] - cu_q[ch];
    if (nq < 0 || nq > seq_lens[ch]) return ORC_ERR_LEN;
  }
  int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < (int64_t)num_chunks * num_kv_heads; ++u) {
    int ch = (int)(u / num_kv_heads);
    int g = (int)(u % num_kv_heads);
    int64_t L = seq_lens[ch];
    int64_t nq = (int64_t)cu_q[ch + 1] - cu_q[ch];
    double* K = malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
    double* V = malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * D);
    double* s = malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* qd = malloc(sizeof(double) * D);
    double lse_h;
    if (!K || !V || !s || !qd) {
#pragma omp atomic write
      err = ORC_ERR_NOMEM;
    } else {
      int gs = gather(&c, page_table + (int64_t)ch * max_pages_per_seq, max_pages_per_seq, g, L,
                      K, V);
      if (gs) {
#pragma omp atomic write
        err = gs;
      } else {
        for (int64_t i = 0; i < nq; ++i) {
          int64_t row = cu_q[ch] + i;
          int64_t p = L - nq + i; /* position of this query token */
          for (int h = g * G; h < (g + 1) * G; ++h) {
            for (int d = 0; d < D; ++d)
              qd[d] = bf16_value(q[(row * num_q_heads + h) * D + d]);
            attend_row(qd, K, V, p + 1, D, softmax_scale, s,
                       out + (row * num_q_heads + h) * D, &lse_h);
            if (lse) lse[row * num_q_heads + h] = lse_h;
          }
        }
      }
    }
    free(K);
    free(V);
    free(s);
    free(qd);
  }
  return err;
}

/* ------------------------------------------------------- split and merge */
/*
 * Unnormalised decode partial over the tokens of logical pages
 * [page_begin, page_end) (clipped to the sequence length):
 *   m = max_t s_t,  l = sum_t exp(s_t - m),  acc = sum_t exp(s_t - m) V[t].
 * An empty range gives m = -inf, l = 0, acc = 0.  Output shapes follow
 * oracle_decode: acc [batch][Hq][D], m and l [batch][Hq].
 */
int oracle_decode_partial(const uint8_t* k_pool, const uint8_t* v_pool, const float* k_scale,
                          const float* v_scale, int kv_dtype, int num_pages, int page_size,
                          int num_kv_heads, int head_dim, const uint16_t* q, int num_q_heads,
                          const int32_t* page_table, int max_pages_per_seq,
                          const int32_t* seq_lens, int batch, double softmax_scale,
                          int page_begin, int page_end, double* acc, double* m_out,
                          double* l_out) {
  cache_t c = {(uint8_t*)k_pool, (uint8_t*)v_pool, k_scale, v_scale, kv_dtype, num_pages,
               page_size, num_kv_heads, head_dim};
  int st = check_cache(&c);
  if (st) return st;
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads) return ORC_ERR_ARG;
  const int G = num_q_heads / num_kv_heads;
  const int D = head_dim;
  for (int b = 0; b < batch; ++b) {
    int64_t n = seq_lens[b];
    double* K = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
    double* V = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * D);
    double* qd = malloc(sizeof(double) * D);
    if (!K || !V || !qd) {
      free(K);
      free(V);
      free(qd);
      return ORC_ERR_NOMEM;
    }
    int64_t t0 = (int64_t)page_begin * page_size;
    int64_t t1 = (int64_t)page_end * page_size;
    if (t1 > n) t1 = n;
    for (int g = 0; g < num_kv_heads && !st; ++g) {
      st = gather(&c, page_table + (int64_t)b * max_pages_per_seq, max_pages_per_seq, g, n, K, V);
      for (int h = g * G; h < (g + 1) * G && !st; ++h) {
        int64_t r = (int64_t)b * num_q_heads + h;
        for (int d = 0; d < D; ++d) qd[d] = bf16_value(q[r * D + d]);
        double m = -INFINITY, l = 0.0;
        for (int d = 0; d < D; ++d) acc[r * D + d] = 0.0;
        for (int64_t t = t0; t < t1; ++t) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qd[d] * K[t * D + d];
          double s = softmax_scale * dot;
          if (s > m) m = s;
        }
        for (int64_t t = t0; t < t1; ++t) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qd[d] * K[t * D + d];
          double e = exp(softmax_scale * dot - m);
          l += e;
          for (int d = 0; d < D; ++d) acc[r * D + d] += e * V[t * D + d];
        }
        m_out[r] = m;
        l_out[r] = l;
      }
    }
    free(K);
    free(V);
    free(qd);
    if (st) return st;
  }
  return ORC_OK;
}

/*
 * Merge of split partials (i = 0..n_parts-1) for each of `rows` rows:
 *   M = max_i m_i,  w_i = exp(m_i - M),
 *   out = sum_i w_i acc_i / sum_i w_i l_i,  lse = M + log(sum_i w_i l_i).
 * Parts with m_i = -inf (empty) carry weight 0.  acc: [n_parts][rows][D];
 * m, l: [n_parts][rows].
 */
int oracle_merge(int n_parts, int rows, int head_dim, const double* acc, const double* m,
                 const double* l, double* out, double* lse) {
  if (n_parts < 0 || rows < 0 || head_dim <= 0) return ORC_ERR_ARG;
  for (int r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int i = 0; i < n_parts; ++i)
      if (m[(int64_t)i * rows + r] > M) M = m[(int64_t)i * rows + r];
    double den = 0.0;
    for (int d = 0; d < head_dim; ++d) out[(int64_t)r * head_dim + d] = 0.0;
    if (M == -INFINITY) {
      lse[r] = -INFINITY;
      continue;
    }
    for (int i = 0; i < n_parts; ++i) {
      double mi = m[(int64_t)i * rows + r];
      if (mi == -INFINITY) continue;
      double w = exp(mi - M);
      den += w * l[(int64_t)i * rows + r];
      for (int d = 0; d < head_dim; ++d)
        out[(int64_t)r * head_dim + d] += w * acc[((int64_t)i * rows + r) * head_dim + d];
    }
    for (int d = 0; d < head_dim; ++d) out[(int64_t)r * head_dim + d] /= den;
    lse[r] = M + log(den);
  }
  return ORC_OK;
}
