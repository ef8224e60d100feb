/*
 * paged_kv_runtime.h -- host-side runtime of libpagedkv.so: the page
 * allocator and the in-flight step planner that feed the attention entry
 * points of paged_kv.h.
 *
 * The operation (pages on TensorRT-LLM):
 *  - TensorRT-LLM concept page (compassingai.com), "關鍵機制 / PagedAttention
 *    及 KV 快取管理": KV memory is handed out in fixed-size pages as a
 *    sequence grows, instead of reserving its maximum length up front, and a
 *    per-sequence table maps logical positions to physical pages.
 *  - same page, "執行時執行模型": every step of the in-flight batch admits new
 *    requests, extends running ones by one token (or a prefill chunk), and
 *    frees the pages of requests that finished, for reuse by the next ones.
 *
 * Everything here is plain host code: no CUDA call, no device memory.  The
 * planner writes host arrays in exactly the layout paged_kv_append,
 * paged_decode_attention and paged_prefill_chunk_attention take, so one
 * host->device copy per step moves them.
 *
 * Allocation policy (fixed, so that results are reproducible):
 *  - The free pages form a stack.  At creation it holds page_order[0..N-1]
 *    with page_order[0] on top (page_order NULL = 0, 1, ..., N-1).
 *  - Growing a sequence pops one page per new logical page, in logical order.
 *  - Releasing a sequence pushes its pages back so that its first logical
 *    page ends on top: the next growth reuses them in the same order.
 *  - Growth is all-or-nothing: a request the free stack cannot cover changes
 *    nothing and returns PKV_ERR_NO_PAGES.
 *
 * A pkv_allocator is not thread-safe: one thread drives it.
 */
#ifndef PAGED_KV_RUNTIME_H
#define PAGED_KV_RUNTIME_H

#include <stdint.h>

#include "paged_kv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_allocator pkv_allocator; /* opaque, owned by the caller */

typedef struct pkv_alloc_stats {
  int32_t num_pages;          /* pool size */
  int32_t page_size;          /* tokens per page */
  int32_t max_seqs;           /* sequence slots */
  int32_t max_pages_per_seq;  /* page-table row length */
  int32_t pages_in_use;       /* pages owned by some sequence */
  int32_t peak_pages_in_use;  /* largest pages_in_use seen */
  int32_t live_seqs;          /* slots with length > 0 */
  int64_t tokens_cached;      /* sum of the live lengths */
} pkv_alloc_stats;

/*
 * Create an allocator over num_pages pages of page_size tokens (64 or 128)
 * for max_seqs sequence slots, each up to max_pages_per_seq pages.
 * page_order: optional host int32[num_pages], a permutation of 0..num_pages-1
 * giving the order pages are first handed out (checked; NULL = ascending).
 * Every slot starts empty (length 0, table row all -1).
 * Returns PKV_OK and *out, or PKV_ERR_NULL / PKV_ERR_SHAPE / PKV_ERR_PAGE_SIZE.
 */
int pkv_allocator_create(int32_t num_pages, int32_t page_size, int32_t max_seqs,
                         int32_t max_pages_per_seq, const int32_t* page_order,
                         pkv_allocator** out);

/* Free the allocator (NULL is a no-op). */
void pkv_allocator_destroy(pkv_allocator* a);

/*
 * Make slot `slot` hold new_len tokens: pops ceil(new_len / page_size) minus
 * the pages it has.  new_len must be >= the slot's length and fit
 * max_pages_per_seq pages (else PKV_ERR_SHAPE).  All-or-nothing
 * (PKV_ERR_NO_PAGES).
 */
int pkv_allocator_grow(pkv_allocator* a, int32_t slot, int32_t new_len);

/* Return all pages of `slot` to the free stack; its length becomes 0. */
int pkv_allocator_release(pkv_allocator* a, int32_t slot);

/* Current length of `slot` in *len. */
int pkv_allocator_seq_len(const pkv_allocator* a, int32_t slot, int32_t* len);

/*
 * The page table: host int32 [max_seqs][max_pages_per_seq], row = slot,
 * -1 past a slot's last page.  Valid until the next call that changes the
 * allocator.  NULL for a NULL allocator.
 */
const int32_t* pkv_allocator_table(const pkv_allocator* a);

/* Counters in *out. */
int pkv_allocator_stats(const pkv_allocator* a, pkv_alloc_stats* out);

/*
 * The free stack from top to bottom into out[0..n-1], n = num_pages -
 * pages_in_use (at most `cap` entries written); *count = n.
 */
int pkv_allocator_free_pages(const pkv_allocator* a, int32_t* out, int32_t cap, int32_t* count);

/*
 * Plan one in-flight step.  Row i of the step is slot slots[i] receiving
 * new_tokens[i] >= 1 tokens (1 for a decode row, more for a prefill chunk).
 * Grows every slot (all-or-nothing over the whole step: on PKV_ERR_NO_PAGES
 * nothing changes), then writes, for i < n:
 *   seq_lens_before[i] = length before the step
 *   cu_new[i]          = sum of new_tokens[0..i-1]   (cu_new[n] = the total)
 *   seq_lens_after[i]  = length after the step
 *   table_rows[i][*]   = the slot's page-table row (max_pages_per_seq entries)
 * These are the page_table / seq_lens_before / cu_new_tokens arguments of
 * paged_kv_append and the page_table / seq_lens (after) arguments of the
 * attention calls, for the same row order.  Any output pointer may be NULL.
 * A slot may appear at most once per step (else PKV_ERR_SHAPE).
 */
int pkv_step_plan(pkv_allocator* a, const int32_t* slots, const int32_t* new_tokens, int32_t n,
                  int32_t* seq_lens_before, int32_t* cu_new, int32_t* seq_lens_after,
                  int32_t* table_rows);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_RUNTIME_H */
