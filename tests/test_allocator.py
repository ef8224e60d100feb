"""The host page allocator and step planner (CPU only, no GPU).

* The oracle (``oracle/allocator.py``) is pinned by a trace worked by hand
  from the allocation policy (``tests/golden/allocator_trace.txt``) and by
  invariants under random operations: no page owned twice, owned + free = the
  pool, a slot of length L owns ceil(L / P) pages.
* The library's allocator (``pkv_allocator_*`` / ``pkv_step_plan`` through the
  C ABI) replays the same trace and then matches the oracle bit for bit
  (statuses, page tables, free stacks, lengths, counters) after every
  operation of long random sequences of grows, releases and steps.
"""
import os

import numpy as np
import pytest

from oracle.allocator import NO_PAGES, SHAPE, AllocatorOracle, pages_for

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "allocator_trace.txt")


@pytest.fixture(scope="module")
def pkv():
    import __graft_entry__

    __graft_entry__._builder().build()
    import paged_kv_cache_476_b200 as m

    return m


def _ints(s):
    return [] if s.strip() == "-" else [int(x) for x in s.split(",")]


def _trace():
    lines = [l.strip() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    head = lines[0].split()
    assert head[0] == "init"
    cfg = dict(num_pages=int(head[1]), page_size=int(head[2]), max_seqs=int(head[3]),
               max_pages=int(head[4]), order=_ints(head[6]))
    ops, plan, peak = [], None, None
    for l in lines[1:]:
        if l.startswith("plan"):
            t = l.split()
            plan = dict(before=_ints(t[2]), cu=_ints(t[4]), after=_ints(t[6]),
                        rows=[_ints(r) for r in t[8].split("/")])
        elif l.startswith("peak"):
            peak = int(l.split()[1])
        else:
            lhs, rhs = l.split("->")
            parts = [p.strip() for p in rhs.split(";")]
            ops.append((lhs.split(), int(parts[0]), [_ints(p) for p in parts[1:4]],
                        _ints(parts[4])))
    return cfg, ops, plan, peak


def _parse_step(arg):
    slots, new = zip(*[(int(a), int(b)) for a, b in (p.split(":") for p in arg.split(","))])
    return list(slots), list(new)


class _Lib:
    """The library allocator behind the oracle's interface (for the trace)."""

    def __init__(self, pkv, cfg):
        self.a = pkv.PageAllocator(cfg["num_pages"], cfg["page_size"], cfg["max_seqs"],
                                   cfg["max_pages"], np.array(cfg["order"], np.int32))
        self.max_pages = cfg["max_pages"]

    def grow(self, s, n):
        try:
            return self.a.grow(s, n)
        except Exception as e:  # PagedKVError carries the status
            return e.status

    def release(self, s):
        self.a.release(s)

    def step_plan(self, slots, new):
        try:
            st, plan = self.a.step_plan(slots, new)
        except Exception as e:
            return e.status, None
        if plan is not None:
            plan = {k: v.tolist() for k, v in plan.items()}
        return st, plan

    def slot_pages(self, s):
        row = self.a.table[s]
        return [int(p) for p in row if p >= 0]

    def free_top_first(self):
        return self.a.free_pages().tolist()

    def peak_pages(self):
        return self.a.stats().peak_pages_in_use


class _Orc(AllocatorOracle):
    def slot_pages(self, s):
        return list(self.pages[s])

    def peak_pages(self):
        return self.peak


def _replay(impl, ops, plan_want, peak_want):
    last_plan = None
    for (op, *args), status, slots_want, free_want in ops:
        if op == "grow":
            st = impl.grow(int(args[0]), int(args[1]))
        elif op == "release":
            impl.release(int(args[0]))
            st = 0
        else:
            st, last_plan = impl.step_plan(*_parse_step(args[0]))
        assert st == status, (op, args)
        for s, want in enumerate(slots_want):
            assert impl.slot_pages(s) == want, (op, args, s)
        assert impl.free_top_first() == free_want, (op, args)
    assert last_plan is not None
    assert last_plan["seq_lens_before"] == plan_want["before"]
    assert last_plan["cu_new"] == plan_want["cu"]
    assert last_plan["seq_lens_after"] == plan_want["after"]
    assert [list(r) for r in last_plan["page_table"]] == plan_want["rows"]
    assert impl.peak_pages() == peak_want


def test_oracle_follows_the_hand_worked_trace():
    cfg, ops, plan, peak = _trace()
    o = _Orc(cfg["num_pages"], cfg["page_size"], cfg["max_seqs"], cfg["max_pages"], cfg["order"])
    _replay(o, ops, plan, peak)


def test_library_follows_the_hand_worked_trace(pkv):
    cfg, ops, plan, peak = _trace()
    _replay(_Lib(pkv, cfg), ops, plan, peak)


def _check_invariants(o: AllocatorOracle, num_pages):
    owned = [p for pages in o.pages for p in pages]
    assert len(owned) == len(set(owned)), "a page owned twice"
    assert sorted(owned + o.free) == list(range(num_pages)), "pages lost or duplicated"
    for pages, length in zip(o.pages, o.length):
        assert len(pages) == pages_for(length, o.page_size)


def _random_ops(rng, max_seqs, page_size, max_pages, n_ops):
    for _ in range(n_ops):
        r = rng.random()
        if r < 0.35:
            yield ("grow", int(rng.integers(max_seqs)),
                   int(rng.integers(0, page_size * max_pages + page_size)))
        elif r < 0.55:
            yield ("release", int(rng.integers(max_seqs)))
        else:
            k = int(rng.integers(1, max_seqs + 1))
            slots = rng.permutation(max_seqs)[:k].tolist()
            if rng.random() < 0.05 and k > 1:
                slots[1] = slots[0]  # a duplicate slot: rejected
            new = [int(rng.choice([1, 1, 1, 3, page_size - 1, page_size, 2 * page_size + 5]))
                   for _ in range(k)]
            if rng.random() < 0.03:
                new[0] = 0  # an empty row: rejected
            yield ("step", slots, new)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_oracle_keeps_its_invariants(seed):
    rng = np.random.default_rng(seed)
    num_pages, page_size, max_seqs, max_pages = 40, 64, 6, 12
    o = AllocatorOracle(num_pages, page_size, max_seqs, max_pages, rng.permutation(num_pages))
    for op in _random_ops(rng, max_seqs, page_size, max_pages, 600):
        if op[0] == "grow":
            o.grow(op[1], max(op[2], o.length[op[1]]))
        elif op[0] == "release":
            o.release(op[1])
        else:
            o.step_plan(op[1], op[2])
        _check_invariants(o, num_pages)


@pytest.mark.parametrize("seed,page_size", [(10, 64), (11, 128), (12, 64)])
def test_library_matches_the_oracle_step_by_step(pkv, seed, page_size):
    rng = np.random.default_rng(seed)
    num_pages, max_seqs, max_pages = 50, 7, 10
    order = rng.permutation(num_pages).astype(np.int32)
    o = AllocatorOracle(num_pages, page_size, max_seqs, max_pages, order)
    a = pkv.PageAllocator(num_pages, page_size, max_seqs, max_pages, order)
    lib = _Lib.__new__(_Lib)
    lib.a, lib.max_pages = a, max_pages
    for op in _random_ops(rng, max_seqs, page_size, max_pages, 800):
        if op[0] == "grow":
            want, got = o.grow(op[1], op[2]), lib.grow(op[1], op[2])
            assert got == want, op
        elif op[0] == "release":
            o.release(op[1])
            lib.release(op[1])
        else:
            want_st, want_plan = o.step_plan(op[1], op[2])
            got_st, got_plan = lib.step_plan(op[1], op[2])
            assert got_st == want_st, op
            if want_plan is not None:
                for k in ("seq_lens_before", "cu_new", "seq_lens_after"):
                    assert got_plan[k] == want_plan[k], (op, k)
                assert [list(r) for r in got_plan["page_table"]] == want_plan["page_table"]
        assert a.table.tolist() == o.table()
        assert a.free_pages().tolist() == o.free_top_first()
        assert [a.seq_len(s) for s in range(max_seqs)] == o.length
        st = a.stats()
        assert st.pages_in_use == o.in_use() and st.peak_pages_in_use == o.peak
        assert st.live_seqs == sum(l > 0 for l in o.length)
        assert st.tokens_cached == sum(o.length)


def test_allocator_rejects_bad_arguments(pkv):
    with pytest.raises(pkv.PagedKVError):
        pkv.PageAllocator(8, 32, 2, 4)  # page size
    with pytest.raises(pkv.PagedKVError):
        pkv.PageAllocator(4, 64, 2, 4, np.array([0, 1, 1, 3], np.int32))  # not a permutation
    with pytest.raises(pkv.PagedKVError):
        pkv.PageAllocator(0, 64, 2, 4)
    a = pkv.PageAllocator(8, 64, 2, 4)
    assert a.grow(0, 100) == 0
    with pytest.raises(pkv.PagedKVError):
        a.grow(0, 50)  # shrinking
    with pytest.raises(pkv.PagedKVError):
        a.grow(2, 1)  # slot out of range
    with pytest.raises(pkv.PagedKVError):
        a.step_plan([0, 0], [1, 1])  # duplicate slot
    assert a.seq_len(0) == 100 and a.table[0].tolist() == [0, 1, -1, -1]


def test_paged_reservation_beats_max_length_reservation(pkv):
    # the point of paging: pages in use track the live lengths, not the maximum
    rng = np.random.default_rng(5)
    P, max_len, slots = 64, 8192, 64
    a = pkv.PageAllocator(slots * max_len // P, P, slots, max_len // P)
    lens = rng.integers(128, 4097, size=slots)
    for s, n in enumerate(lens):
        assert a.grow(s, int(n)) == 0
    st = a.stats()
    assert st.pages_in_use == sum(pages_for(int(n), P) for n in lens)
    assert st.pages_in_use < 0.6 * slots * (max_len // P)
