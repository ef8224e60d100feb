/*
 * paged_kv.h -- C ABI of libpagedkv.so: attention over a paged KV cache for an
 * in-flight batch, on NVIDIA B200 (sm_100a).
 *
 * The operation (pages on TensorRT-LLM):
 *  - TensorRT-LLM concept page (compassingai.com), "關鍵機制 / PagedAttention
 *    及 KV 快取管理": each sequence's K/V lives in fixed-size pages (64 or 128
 *    tokens); a per-sequence page table maps logical token positions to
 *    physical pages, so no maximum length is reserved up front.
 *  - same page, "技術原理 / 編譯期圖最佳化": page-table lookups sit on every KV
 *    read and write of the attention operator.
 *  - same page, "執行時執行模型": each forward pass of the in-flight batch
 *    appends the new tokens' K/V and attends over the pages.
 *  - same page, "關鍵效能引數": context (prefill) tokens are processed in
 *    parallel over the paged cache.
 *  - yololab.net guide, "FP8 與極致量化": FP8 storage halves the bytes moved.
 *
 * Conventions shared by every entry point:
 *  - All array pointers are DEVICE memory owned by the caller; the library
 *    allocates nothing and keeps no state between calls.
 *  - Pools: separate K and V pools, each [num_pages][num_kv_heads][page_size]
 *    [head_dim], row-major, element type bf16 or FP8 E4M3 (1 byte).  Base
 *    addresses must be 16-byte aligned.
 *  - Scales of the one-byte and FP4 pools: one fp32 per (page, kv head) for
 *    K and one for V, layout [num_pages][num_kv_heads]; the stored value of
 *    an E4M3 element is decode_e4m3(code) * scale.  Scales must be finite
 *    and in (0, 2^15].
 *    The caller chooses them (e.g. absmax/448 of what the page will hold);
 *    the library reads them and never updates them.
 *  - INT8 pools: code = nearest integer (ties to even) of fp32(x) / scale,
 *    clamped to +-127 (NaN stored as 0); stored value = code * scale.
 *  - FP4 pools (PKV_KV_NVFP4; solosoft post, FAQ: FP4 quantisation on
 *    Blackwell).  Each pool is ONE buffer of rows * (head_dim/2 + head_dim/16)
 *    bytes, rows = num_pages * num_kv_heads * page_size, row index
 *    (page * num_kv_heads + kv_head) * page_size + slot:
 *      codes   [rows][head_dim/2]   two E2M1 codes per byte, the even element
 *                                    in the low nibble;
 *      blocks  [rows][head_dim/16]  one E4M3 block scale per 16 consecutive
 *                                    elements of a row, after all the codes.
 *    With s the (page, kv head) fp32 scale and amax the largest |x| of a
 *    block: sb = e4m3_rne_satfinite(amax / fp32(6 * s)), d = fp32(decode(sb) * s),
 *    code = e2m1_rne_satfinite(x / d) (0 when d = 0, +0 for NaN); stored
 *    value = e2m1(code) * decode(sb) * s.  The caller picks s (e.g.
 *    absmax / (448 * 6) of what the page will hold).
 *  - Page table: int32 [batch][max_pages_per_seq], row-major; entry j holds the
 *    physical page of tokens [j*page_size, (j+1)*page_size).  Entries past the
 *    last page a sequence needs are ignored (-1 by convention).
 *  - GQA: q head h reads kv head h / gqa_group (contiguous groups).
 *  - Supported: page_size in {64, 128}; head_dim in {64, 128};
 *    gqa_group in {1, 2, 4, 8}; bf16 Q/K/V/out; K/V pools bf16, E4M3, INT8
 *    or FP4.
 *  - Asynchronous: a call validates its arguments on the host, returns a
 *    negative pkv_status before launching anything if they are wrong, and
 *    otherwise enqueues its kernels on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and returns PKV_OK.  Launch failures return
 *    PKV_ERR_CUDA.  Data-dependent errors (bad page ids, lengths past the page
 *    table, a bounded wait that gave up) are detected on the device: the
 *    offending tokens are skipped and, when cache->error_flags is non-NULL,
 *    the matching PKV_FLAG_* bit is OR-ed into it.  Kernels never trap.
 *  - Not done by the library: page allocation (the caller owns the pool and
 *    the table), positional encoding (K arrives post-rotary), scale choice.
 */
#ifndef PAGED_KV_H
#define PAGED_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PKV_OK = 0,
  PKV_ERR_NULL = -1,        /* a required pointer is NULL */
  PKV_ERR_SHAPE = -2,       /* a count or size is negative or inconsistent */
  PKV_ERR_PAGE_SIZE = -3,   /* page_size not in {64, 128} */
  PKV_ERR_HEAD_DIM = -4,    /* head_dim not in {64, 128} */
  PKV_ERR_GQA = -5,         /* num_q_heads != gqa_group*num_kv_heads, or group unsupported */
  PKV_ERR_DTYPE = -6,       /* unknown kv_dtype, or a quantised pool without scales */
  PKV_ERR_WORKSPACE = -7,   /* decode workspace NULL, misaligned or too small */
  PKV_ERR_CUDA = -8,        /* a CUDA runtime call or kernel launch failed */
  PKV_ERR_ALIGN = -9,       /* a pointer that must be 16-byte aligned is not */
  PKV_ERR_UNSUPPORTED = -10, /* a valid combination this build does not implement */
  PKV_ERR_SCRATCH_LIMIT = -11, /* request needs more than the static decode scratch */
  PKV_ERR_NO_PAGES = -12     /* the free pages cannot cover a growth (paged_kv_runtime.h) */
} pkv_status;

typedef enum {
  PKV_KV_BF16 = 0,     /* bf16 elements */
  PKV_KV_FP8_E4M3 = 1, /* one E4M3 code per element, per-(page, kv head) fp32 scale */
  PKV_KV_INT8 = 2,     /* one INT8 code per element (+-127), per-(page, kv head) scale */
  PKV_KV_NVFP4 = 3     /* E2M1 codes, an E4M3 scale per 16 elements, per-(page, kv head)
                          scale: see "FP4 pools" above */
} pkv_kv_dtype;

/* Device-side error bits OR-ed into pkv_cache.error_flags. */
#define PKV_FLAG_BAD_PAGE 0x1    /* a page-table entry outside [0, num_pages) */
#define PKV_FLAG_BAD_LENGTH 0x2  /* a length < 0, past max_pages_per_seq*page_size, or a
                                    chunk longer than its sequence */
#define PKV_FLAG_TIMEOUT 0x4     /* a bounded wait inside a kernel gave up */
#define PKV_FLAG_BAD_SCALE 0x8   /* an FP8 scale outside (0, 2^15] */

/* The paged KV cache: pools, optional FP8 scales, geometry. */
typedef struct pkv_cache {
  void* k_pool;          /* [num_pages][num_kv_heads][page_size][head_dim] (FP4: codes,
                            then block scales, as above) */
  void* v_pool;          /* same shape as k_pool */
  const float* k_scale;  /* [num_pages][num_kv_heads] fp32; NULL for bf16 pools */
  const float* v_scale;  /* [num_pages][num_kv_heads] fp32; NULL for bf16 pools */
  int32_t num_pages;     /* >= 1 */
  int32_t page_size;     /* tokens per page: 64 or 128 */
  int32_t num_kv_heads;  /* >= 1 */
  int32_t head_dim;      /* 64 or 128 */
  int32_t kv_dtype;      /* pkv_kv_dtype */
  int32_t* error_flags;  /* optional device int32; NULL disables reporting */
} pkv_cache;

/*
 * Paged KV append (the paged store).  Writes the K/V of this step's new tokens
 * into their pages: new token j of sequence b sits at logical position
 * pos = seq_lens_before[b] + (j - cu_new_tokens[b]) and is stored in page
 * page_table[b][pos / page_size], slot pos % page_size.  bf16 pools receive
 * the input bits unchanged; E4M3 pools receive
 * e4m3_round_nearest_even_satfinite(fp32(x) / scale[page][kv_head]) with an
 * IEEE fp32 division; INT8 and FP4 pools the codes defined above (FP4: a
 * token's row is quantised block by block, its block scales included).  Source: concept page "PagedAttention 及 KV 快取管理"
 * and "執行時執行模型" (attention updates the KV pages).
 *   page_table        int32 [batch][max_pages_per_seq]
 *   seq_lens_before   int32 [batch], tokens already cached
 *   cu_new_tokens     int32 [batch+1], exclusive prefix sum of new tokens
 *   total_new_tokens  == cu_new_tokens[batch] (host copy, sizes the grid)
 *   k_new, v_new      bf16 [total_new_tokens][num_kv_heads][head_dim]
 * Tokens whose page entry is invalid are skipped (PKV_FLAG_BAD_PAGE).
 */
int paged_kv_append(const pkv_cache* cache, const int32_t* page_table, int32_t max_pages_per_seq,
                    const int32_t* seq_lens_before, const int32_t* cu_new_tokens, int32_t batch,
                    int32_t total_new_tokens, const void* k_new, const void* v_new,
                    void* stream);

/*
 * Split planning for decode (host only, no CUDA calls).  Decode runs as one
 * persistent wave of C CTAs.  The work list is every (sequence, kv head) unit
 * cut into tiles (64 tokens for bf16 and FP4 pools, 128 for E4M3 and INT8, so
 * that a tile is 32 KB of K and V at head_dim 128), concatenated in
 * (sequence, kv head) order; CTA c takes the contiguous range
 * [c*T/C, (c+1)*T/C) of the T tiles, so every CTA streams the same number of
 * KV bytes whatever the length mix (when C > T only T CTAs take work).  A
 * unit that a range boundary cuts becomes several split-KV partials merged
 * in the same launch.  C = num_ctas if num_ctas > 0, else
 * num_sms * ctas_per_sm; C never exceeds the 64-token tiles of the largest
 * batch the arguments allow.
 * Output: *out_ctas = C >= 1.
 */
int paged_decode_plan(int32_t batch, int32_t num_kv_heads, int32_t max_seq_len,
                      int32_t num_sms, int32_t num_ctas, int32_t ctas_per_sm,
                      int32_t* out_ctas);

/*
 * Bytes of decode workspace for these arguments, sized for the current
 * device (call it with the device that will run the decode current).
 * Returns 0 on bad arguments.  The workspace holds the split partials
 * ((units + C) slots of G x (head_dim + 2) floats, units = batch *
 * num_kv_heads) and one (first slot, segment count) record per unit.  It
 * needs no initialisation: every call writes each value it later reads.
 * Calls that share a workspace must not overlap on the GPU.
 */
size_t paged_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t max_seq_len, int32_t num_ctas);

/*
 * Split-KV decode attention: one query token per sequence attends over all
 * seq_lens[b] tokens of its pages.  For q head h (kv head g = h / gqa_group):
 *   s_t = softmax_scale * q[b][h] . K_b[t],   t < seq_lens[b]
 *   out[b][h] = sum_t exp(s_t - m) V_b[t] / sum_t exp(s_t - m)   (bf16)
 *   lse[b][h] = m + ln(sum_t exp(s_t - m))                       (fp32)
 * computed as online-softmax partials over page ranges (see
 * paged_decode_plan); the pieces of a (sequence, kv head) cut across CTAs
 * are merged by a second kernel enqueued by the same call (a programmatic
 * dependent launch, so its launch overlaps the first).  A sequence of length 0
 * yields out = 0 and lse = -inf.  Source: concept page "執行時執行模型"
 * (attention reads the KV pages each step) and "PagedAttention 及 KV 快取管理".
 *   q             bf16 [batch][num_q_heads][head_dim]
 *   seq_lens      int32 [batch], tokens per sequence AFTER this step's append
 *   max_seq_len   host upper bound of seq_lens (plans the grid)
 *   out           bf16 [batch][num_q_heads][head_dim]
 *   lse           fp32 [batch][num_q_heads], or NULL
 *   workspace     16-byte aligned, >= paged_decode_workspace_bytes(...) bytes
 *   num_ctas      0 = automatic plan; > 0 forces the CTA count (see plan)
 */
int paged_decode_attention(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                           int32_t gqa_group, const int32_t* page_table,
                           int32_t max_pages_per_seq, const int32_t* seq_lens, int32_t batch,
                           int32_t max_seq_len, float softmax_scale, void* out, float* lse,
                           void* workspace, size_t workspace_bytes, int32_t num_ctas,
                           void* stream);

/*
 * Decode step with the append fused in: one launch stores each sequence's
 * new token and attends over all its tokens, the new one included.  Same
 * arguments and result as paged_decode_attention, plus the new tokens:
 *   k_new, v_new  bf16 [batch][num_kv_heads][head_dim], 16-byte aligned; row b
 *                 is sequence b's new token, stored at position
 *                 seq_lens[b] - 1 (seq_lens counts it)
 * The pools end up holding exactly the bytes of
 *   paged_kv_append(cache, page_table, max_pages_per_seq,
 *                   seq_lens_before = seq_lens - 1, cu_new = 0, 1, ..., batch, ...)
 * (bf16 bits; E4M3 or INT8 codes of x / scale with the page's scales), and out
 * and lse are those of paged_decode_attention on that cache.  The token is
 * stored by the CTA that reads the tile holding it, which then orders the
 * stores before its own tile loads; the new K/V therefore make one trip
 * through L2 instead of a separate kernel's.  Rows with seq_lens[b] = 0 store
 * nothing.  A row whose length exceeds max_pages_per_seq * page_size, or
 * whose page id is invalid, stores nothing and sets the error flag, as the
 * decode does.  Source: concept page "PagedAttention 及 KV 快取管理" (each
 * step appends the token's K/V to the sequence's pages, then attention reads
 * them) and "編譯期圖最佳化" (the paged operations fused into the engine).
 * Errors: PKV_ERR_NULL for a missing k_new / v_new, PKV_ERR_ALIGN for a
 * misaligned one, then every check of paged_decode_attention.
 */
int paged_decode_attention_append(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                                  int32_t gqa_group, const int32_t* page_table,
                                  int32_t max_pages_per_seq, const int32_t* seq_lens,
                                  int32_t batch, int32_t max_seq_len, float softmax_scale,
                                  const void* k_new, const void* v_new, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, int32_t num_ctas,
                                  void* stream);

/*
 * Causal prefill-chunk attention over the paged cache.  Chunk c owns the
 * queries [cu_q_lens[c], cu_q_lens[c+1]) of the packed q and has seq_lens[c]
 * tokens cached AFTER its append (its own new tokens included).  Query i of a
 * chunk with n queries sits at position p = seq_lens[c] - n + i and attends to
 * keys 0..p inclusive:
 *   out[row][h] = softmax_t<=p(softmax_scale * q[row][h] . K_c[t]) V_c   (bf16)
 *   lse[row][h] = ln sum_t<=p exp(softmax_scale * q[row][h] . K_c[t])    (fp32)
 * QK^T and PV run on the tcgen05 tensor cores.  Source: concept page
 * "關鍵效能引數" (context tokens processed in parallel over pages, with
 * FlashAttention) and ab123.xyz post (FA-2 with PagedAttention for long
 * sequences) -- both prior art; this is an sm_100a design.
 *   q          bf16 [total_q][num_q_heads][head_dim], total_q = cu_q_lens[num_chunks]
 *   cu_q_lens  int32 [num_chunks+1]
 *   page_table int32 [num_chunks][max_pages_per_seq]
 *   seq_lens   int32 [num_chunks]
 *   total_q    host copy of cu_q_lens[num_chunks] (rows of q and out)
 *   max_q_len  host upper bound of any chunk's query count (plans the grid)
 * E4M3 pools are converted tile by tile to bf16 in shared memory (exact) and
 * their per-(page, head) scales applied to the scores (K) and to P (V).
 *   out        bf16 [total_q][num_q_heads][head_dim]
 *   lse        fp32 [total_q][num_q_heads], or NULL
 */
int paged_prefill_chunk_attention(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                                  int32_t gqa_group, const int32_t* cu_q_lens,
                                  const int32_t* page_table, int32_t max_pages_per_seq,
                                  const int32_t* seq_lens, int32_t num_chunks, int32_t total_q,
                                  int32_t max_q_len, float softmax_scale, void* out, float* lse,
                                  void* stream);

/*
 * Decode attention without any device allocation.  The pages have no
 * counterpart: this entry point exists for callers that cannot call
 * cudaMalloc or take memory from an allocator (code handed only input and
 * output pointers by a host framework or plugin interface, code running where
 * allocation is forbidden, or code that must not change the device's
 * allocation state).  It computes exactly what paged_decode_attention
 * computes, with the same arguments minus the workspace: the split partials
 * and per-unit records live in a scratch array inside the library, a file-scope
 * __device__ array of PKV_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU which
 * loads the library holds until the process exits.
 *  - Sizes whose workspace (paged_decode_workspace_bytes) exceeds the array
 *    are rejected with PKV_ERR_SCRATCH_LIMIT before anything is enqueued.
 *  - Nothing in the array needs to start at zero: each call writes every
 *    value it later reads.  A call allocates nothing and calls no allocating
 *    library routine.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents: calls whose executions overlap on the GPU (unordered streams)
 *    race and give wrong results.  Order them on one stream.
 *  - The first call on a device looks up the array's device address with that
 *    device current; make that first call before any stream capture.
 *  - Under CUDA's default lazy module loading the array's memory is committed
 *    by that first call on each device, so the first call is the one that
 *    can fail for lack of device memory (PKV_ERR_CUDA).  Make one call while
 *    memory is still free, or set CUDA_MODULE_LOADING=EAGER, before handing
 *    the device's memory to another allocator.
 *  - The address is cached per device for the life of the process and does
 *    not survive cudaDeviceReset: do not call this entry point after a reset.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)
int paged_decode_attention_noalloc(const pkv_cache* cache, const void* q, int32_t num_q_heads,
                                   int32_t gqa_group, const int32_t* page_table,
                                   int32_t max_pages_per_seq, const int32_t* seq_lens,
                                   int32_t batch, int32_t max_seq_len, float softmax_scale,
                                   void* out, float* lse, int32_t num_ctas, void* stream);

/*
 * Combine attention results over disjoint key ranges (sequence parallelism).
 * Part r attended over its own keys of each row -- e.g. one GPU's pages of a
 * long sequence, via paged_decode_attention with that GPU's slice of the page
 * table -- and gave the normalised output out_r and its lse_r.  The result
 * over all keys is
 *   lse = log sum_r exp(lse_r),   out = sum_r exp(lse_r - lse) out_r,
 * the split-KV reduction (concept page, "執行時執行模型": attention over the
 * sequence's pages; splitting them across devices is this library's reading).
 * A part with lse_r = -inf (no key) has weight 0; a row whose parts are all
 * empty becomes 0 with lse -inf.
 *   parts      bf16 [num_parts][rows][head_dim], 16-byte aligned
 *   lse_parts  fp32 [num_parts][rows]
 *   out        bf16 [rows][head_dim], 16-byte aligned; lse fp32 [rows] or NULL
 * rows = batch * num_q_heads.  head_dim in {64, 128}; num_parts >= 1.
 */
int paged_attention_combine(const void* parts, const float* lse_parts, int32_t num_parts,
                            int32_t rows, int32_t head_dim, void* out, float* lse,
                            void* stream);

/*
 * Check of the bounded waits (failure detection without a fault).  Every wait
 * inside this library's kernels (a TMA tile landing, a ring slot freed, a
 * tensor-core product done) gives up after a time limit, ORs
 * PKV_FLAG_TIMEOUT into cache->error_flags and lets the kernel return, so a
 * lost arrival ends in a status the host reads and the context stays usable.
 * This call enqueues one CTA that runs that same wait on an mbarrier nothing
 * arrives on, with no copy or tensor-core operation in flight.  Source: the
 * murmur post's evaluation criteria, which list fault recovery (故障恢復).
 *   error_flags  device int32; PKV_FLAG_TIMEOUT is OR-ed in when the wait gives up
 *   limit_ns     how long to wait: 0 = the limit the kernels use (2 s);
 *                at most that limit, else PKV_ERR_SHAPE
 *   waited_ns    optional device int64: the time waited (-1 if it was not cut off)
 * Returns PKV_ERR_NULL without error_flags, PKV_ERR_CUDA if the launch fails.
 */
int pkv_check_bounded_wait(int32_t* error_flags, int64_t limit_ns, int64_t* waited_ns,
                           void* stream);

/* Human-readable name of a pkv_status value (static storage). */
const char* pkv_status_string(int status);

/* ABI version of this library: (major << 16) | minor. */
int pkv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_H */
