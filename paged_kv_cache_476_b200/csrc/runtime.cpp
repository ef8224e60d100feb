// Host-side page allocator and in-flight step planner (no CUDA).
//
// TensorRT-LLM concept page, "PagedAttention 及 KV 快取管理": pages are
// handed out as sequences grow and returned when they finish; "執行時執行模型":
// each step of the in-flight batch extends running sequences and admits new
// ones.  The allocator owns a stack of free page ids, one length per slot and
// the page table itself (row = slot), so a step's arguments for the kernels
// are a row gather away.
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "../../include/paged_kv_runtime.h"

struct pkv_allocator {
  int32_t num_pages, page_size, max_seqs, max_pages;
  std::vector<int32_t> free_stack;  // back() = top
  std::vector<int32_t> len;         // [max_seqs]
  std::vector<int32_t> table;       // [max_seqs][max_pages], -1 past the last page
  int32_t in_use = 0, peak = 0;
  std::vector<int32_t> mark;        // step-plan scratch: slot seen in this step
};

namespace {

int64_t pages_for(int64_t len, int32_t page_size) { return (len + page_size - 1) / page_size; }

}  // namespace

extern "C" int pkv_allocator_create(int32_t num_pages, int32_t page_size, int32_t max_seqs,
                                    int32_t max_pages_per_seq, const int32_t* page_order,
                                    pkv_allocator** out) {
  if (!out) return PKV_ERR_NULL;
  *out = nullptr;
  if (page_size != 64 && page_size != 128) return PKV_ERR_PAGE_SIZE;
  if (num_pages < 1 || max_seqs < 1 || max_pages_per_seq < 1) return PKV_ERR_SHAPE;
  if ((int64_t)max_seqs * max_pages_per_seq > ((int64_t)1 << 31) - 1) return PKV_ERR_SHAPE;
  if (page_order) {  // must be a permutation
    std::vector<uint8_t> seen((size_t)num_pages, 0);
    for (int32_t i = 0; i < num_pages; ++i) {
      const int32_t p = page_order[i];
      if (p < 0 || p >= num_pages || seen[(size_t)p]) return PKV_ERR_SHAPE;
      seen[(size_t)p] = 1;
    }
  }
  pkv_allocator* a = new (std::nothrow) pkv_allocator;
  if (!a) return PKV_ERR_SHAPE;
  a->num_pages = num_pages;
  a->page_size = page_size;
  a->max_seqs = max_seqs;
  a->max_pages = max_pages_per_seq;
  a->free_stack.resize((size_t)num_pages);
  for (int32_t i = 0; i < num_pages; ++i)  // page_order[0] on top
    a->free_stack[(size_t)(num_pages - 1 - i)] = page_order ? page_order[i] : i;
  a->len.assign((size_t)max_seqs, 0);
  a->table.assign((size_t)max_seqs * max_pages_per_seq, -1);
  a->mark.assign((size_t)max_seqs, 0);
  *out = a;
  return PKV_OK;
}

extern "C" void pkv_allocator_destroy(pkv_allocator* a) { delete a; }

extern "C" int pkv_allocator_grow(pkv_allocator* a, int32_t slot, int32_t new_len) {
  if (!a) return PKV_ERR_NULL;
  if (slot < 0 || slot >= a->max_seqs) return PKV_ERR_SHAPE;
  const int32_t old_len = a->len[(size_t)slot];
  if (new_len < old_len) return PKV_ERR_SHAPE;
  const int64_t have = pages_for(old_len, a->page_size);
  const int64_t need = pages_for(new_len, a->page_size);
  if (need > a->max_pages) return PKV_ERR_SHAPE;
  if (need - have > (int64_t)a->free_stack.size()) return PKV_ERR_NO_PAGES;
  int32_t* row = a->table.data() + (size_t)slot * a->max_pages;
  for (int64_t j = have; j < need; ++j) {
    row[j] = a->free_stack.back();
    a->free_stack.pop_back();
  }
  a->in_use += (int32_t)(need - have);
  if (a->in_use > a->peak) a->peak = a->in_use;
  a->len[(size_t)slot] = new_len;
  return PKV_OK;
}

extern "C" int pkv_allocator_release(pkv_allocator* a, int32_t slot) {
  if (!a) return PKV_ERR_NULL;
  if (slot < 0 || slot >= a->max_seqs) return PKV_ERR_SHAPE;
  const int64_t have = pages_for(a->len[(size_t)slot], a->page_size);
  int32_t* row = a->table.data() + (size_t)slot * a->max_pages;
  for (int64_t j = have - 1; j >= 0; --j) {  // first logical page ends on top
    a->free_stack.push_back(row[j]);
    row[j] = -1;
  }
  a->in_use -= (int32_t)have;
  a->len[(size_t)slot] = 0;
  return PKV_OK;
}

extern "C" int pkv_allocator_seq_len(const pkv_allocator* a, int32_t slot, int32_t* len) {
  if (!a || !len) return PKV_ERR_NULL;
  if (slot < 0 || slot >= a->max_seqs) return PKV_ERR_SHAPE;
  *len = a->len[(size_t)slot];
  return PKV_OK;
}

extern "C" const int32_t* pkv_allocator_table(const pkv_allocator* a) {
  return a ? a->table.data() : nullptr;
}

extern "C" int pkv_allocator_stats(const pkv_allocator* a, pkv_alloc_stats* out) {
  if (!a || !out) return PKV_ERR_NULL;
  out->num_pages = a->num_pages;
  out->page_size = a->page_size;
  out->max_seqs = a->max_seqs;
  out->max_pages_per_seq = a->max_pages;
  out->pages_in_use = a->in_use;
  out->peak_pages_in_use = a->peak;
  int32_t live = 0;
  int64_t tokens = 0;
  for (int32_t l : a->len) {
    live += l > 0;
    tokens += l;
  }
  out->live_seqs = live;
  out->tokens_cached = tokens;
  return PKV_OK;
}

extern "C" int pkv_allocator_free_pages(const pkv_allocator* a, int32_t* out, int32_t cap,
                                        int32_t* count) {
  if (!a || !count) return PKV_ERR_NULL;
  if (cap < 0 || (cap > 0 && !out)) return PKV_ERR_SHAPE;
  const int32_t n = (int32_t)a->free_stack.size();
  for (int32_t i = 0; i < n && i < cap; ++i) out[i] = a->free_stack[(size_t)(n - 1 - i)];
  *count = n;
  return PKV_OK;
}

extern "C" int pkv_step_plan(pkv_allocator* a, const int32_t* slots, const int32_t* new_tokens,
                             int32_t n, int32_t* seq_lens_before, int32_t* cu_new,
                             int32_t* seq_lens_after, int32_t* table_rows) {
  if (!a) return PKV_ERR_NULL;
  if (n < 0) return PKV_ERR_SHAPE;
  if (n > 0 && (!slots || !new_tokens)) return PKV_ERR_NULL;
  // validate the whole step before changing anything
  int64_t pages_needed = 0, total = 0;
  int st = PKV_OK;
  for (int32_t i = 0; i < n && st == PKV_OK; ++i) {
    const int32_t s = slots[i];
    if (s < 0 || s >= a->max_seqs || a->mark[(size_t)s] || new_tokens[i] < 1) {
      st = PKV_ERR_SHAPE;
      break;
    }
    a->mark[(size_t)s] = 1;
    const int64_t old_len = a->len[(size_t)s];
    const int64_t new_len = old_len + new_tokens[i];
    const int64_t need = pages_for(new_len, a->page_size);
    if (new_len > INT32_MAX || need > a->max_pages) st = PKV_ERR_SHAPE;
    pages_needed += need - pages_for(old_len, a->page_size);
    total += new_tokens[i];
  }
  for (int32_t i = 0; i < n; ++i)  // clear the marks set above
    if (slots[i] >= 0 && slots[i] < a->max_seqs) a->mark[(size_t)slots[i]] = 0;
  if (st != PKV_OK) return st;
  if (total > INT32_MAX) return PKV_ERR_SHAPE;
  if (pages_needed > (int64_t)a->free_stack.size()) return PKV_ERR_NO_PAGES;
  int32_t cu = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int32_t s = slots[i];
    const int32_t before = a->len[(size_t)s];
    pkv_allocator_grow(a, s, before + new_tokens[i]);  // cannot fail: checked above
    if (seq_lens_before) seq_lens_before[i] = before;
    if (cu_new) cu_new[i] = cu;
    if (seq_lens_after) seq_lens_after[i] = before + new_tokens[i];
    if (table_rows)
      memcpy(table_rows + (size_t)i * a->max_pages, a->table.data() + (size_t)s * a->max_pages,
             sizeof(int32_t) * (size_t)a->max_pages);
    cu += new_tokens[i];
  }
  if (cu_new) cu_new[n] = cu;
  return PKV_OK;
}
