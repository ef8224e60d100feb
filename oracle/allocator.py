"""Oracle of the page allocator and step planner (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module; it shares no code with the library.

What it follows (TensorRT-LLM concept page, "關鍵機制 / PagedAttention 及 KV
快取管理": pages are handed out as a sequence grows and a per-sequence table
maps logical positions to them; "執行時執行模型": finished requests return
their pages for the next ones).  The pages fix no order of reuse; the library
documents one, and this is that policy written out step by step:

* free pages are a stack; at creation ``page_order[0]`` is on top;
* growing a sequence pops one page per new logical page, in logical order;
* releasing a sequence pushes its pages back, last logical page first, so the
  first logical page ends on top;
* a growth (or a whole step) that the free stack cannot cover changes nothing.

Plain Python lists, no cleverness: the state after every operation can be
checked by eye against the rules above.
"""
from __future__ import annotations

NO_PAGES = -12
SHAPE = -2


def pages_for(length: int, page_size: int) -> int:
    """Pages that hold ``length`` tokens: ceil(length / page_size)."""
    return -(-length // page_size)


class AllocatorOracle:
    def __init__(self, num_pages, page_size, max_seqs, max_pages_per_seq, page_order=None):
        order = list(range(num_pages)) if page_order is None else [int(p) for p in page_order]
        self.page_size = page_size
        self.max_pages = max_pages_per_seq
        self.free = list(reversed(order))  # free[-1] is the top of the stack
        self.pages = [[] for _ in range(max_seqs)]  # logical page list per slot
        self.length = [0] * max_seqs
        self.peak = 0

    # state --------------------------------------------------------------
    def in_use(self) -> int:
        return sum(len(p) for p in self.pages)

    def table(self):
        """Page table rows, -1 past the last page."""
        return [p + [-1] * (self.max_pages - len(p)) for p in self.pages]

    def free_top_first(self):
        return list(reversed(self.free))

    # operations ---------------------------------------------------------
    def grow(self, slot, new_len) -> int:
        if new_len < self.length[slot]:
            return SHAPE
        need = pages_for(new_len, self.page_size)
        if need > self.max_pages:
            return SHAPE
        extra = need - len(self.pages[slot])
        if extra > len(self.free):
            return NO_PAGES
        for _ in range(extra):
            self.pages[slot].append(self.free.pop())
        self.length[slot] = new_len
        self.peak = max(self.peak, self.in_use())
        return 0

    def release(self, slot):
        for page in reversed(self.pages[slot]):
            self.free.append(page)
        self.pages[slot] = []
        self.length[slot] = 0

    def step_plan(self, slots, new_tokens):
        """(status, plan) like the library's step planner."""
        if len(set(slots)) != len(slots) or any(n < 1 for n in new_tokens):
            return SHAPE, None
        extra = 0
        for s, n in zip(slots, new_tokens):
            need = pages_for(self.length[s] + n, self.page_size)
            if need > self.max_pages:
                return SHAPE, None
            extra += need - len(self.pages[s])
        if extra > len(self.free):
            return NO_PAGES, None
        before, after, cu, rows = [], [], [0], []
        for s, n in zip(slots, new_tokens):
            before.append(self.length[s])
            self.grow(s, self.length[s] + n)
            after.append(self.length[s])
            cu.append(cu[-1] + n)
            rows.append(self.table()[s])
        return 0, {"seq_lens_before": before, "cu_new": cu, "seq_lens_after": after,
                   "page_table": rows}
