"""An in-flight batch driven step by step through the library (needs a GPU).

Requests arrive, are prefilled in chunks, decode token by token, finish and
free their pages, which later requests reuse.  Every step plans its pages
with the library's host planner (``pkv_step_plan``), then runs the library's
append, decode and prefill kernels through ``StepDriver``.  The reference for
each step is the oracle over every request's whole K/V history laid out
contiguously (one page per request, identity table): the paging of the
library plays no part in it, so a wrong page, a stale page after reuse or a
lost token shows up as an attention mismatch (max-abs 1e-2, mean-abs 1e-3,
lse 2e-3 against fp64).  The pool is small enough that admission has to wait
for pages, so the NO_PAGES path and page reuse are exercised.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.allocator import pages_for
from tests._gpu import compare

pytestmark = pytest.mark.gpu


def _bits(t):
    return oracle.bf16_bits(t.cpu())


def _reference(hist_k, hist_v, rows, lens, q, cu_q, P_ref, Hkv, D, scale, kind):
    """Oracle attention over contiguous histories: row i owns page i."""
    n = len(rows)
    c = oracle.Cache(n, P_ref, Hkv, D, "bf16")
    table = np.arange(n, dtype=np.int32).reshape(n, 1)
    for i, (r, L) in enumerate(zip(rows, lens)):
        c.append(table[i:i + 1], np.zeros(1, np.int32), np.array([0, L], np.int32),
                 _bits(hist_k[r][:L]), _bits(hist_v[r][:L]))
    if kind == "decode":
        return c.decode(_bits(q), table, np.array(lens, np.int32), scale)
    return c.prefill_chunk(_bits(q), np.array(cu_q, np.int32), table, np.array(lens, np.int32),
                           scale)


@pytest.mark.parametrize("page_size", [64, 128])
def test_inflight_batch_matches_contiguous_oracle(page_size):
    import paged_kv_cache_476_b200 as pkv

    rng = np.random.default_rng(40 + page_size)
    gen = torch.Generator().manual_seed(41 + page_size)
    Hq, Hkv, D = 8, 2, 128
    scale = D ** -0.5
    n_req, slots = 14, 6
    prompt = rng.integers(1, 400, size=n_req)
    decode_tokens = rng.integers(1, 9, size=n_req)
    total = prompt + decode_tokens
    max_len = int(total.max())
    P_ref = max_len  # oracle: one page holds a whole request
    hist_k = [torch.randn(int(t), Hkv, D, generator=gen).to(torch.bfloat16) for t in total]
    hist_v = [torch.randn(int(t), Hkv, D, generator=gen).to(torch.bfloat16) for t in total]
    # a pool of under half of what all slots at their longest would need
    num_pages = int(0.45 * slots * pages_for(max_len, page_size)) + 2
    max_pages = pages_for(max_len, page_size)
    k_pool = torch.full((num_pages, Hkv, page_size, D), float("nan"), dtype=torch.bfloat16,
                        device="cuda")
    v_pool = torch.full_like(k_pool, float("nan"))
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = pkv.PagedKVCache(k_pool, v_pool, "bf16", None, None, flags)
    alloc = pkv.PageAllocator(num_pages, page_size, slots, max_pages,
                              rng.permutation(num_pages).astype(np.int32))
    drv = pkv.StepDriver(cache, alloc, max_rows=slots)

    chunk_cap = 96
    waiting = list(range(n_req))
    slot_of, done_tok = {}, {}  # request -> slot, tokens already in the cache
    free_slots = list(range(slots))
    admitted = {}  # request -> admission number (a re-admission gets a new one)
    n_admissions = steps = no_pages = checked = 0
    admit = True
    while waiting or slot_of:
        steps += 1
        assert steps < 400
        while admit and waiting and free_slots:  # admit in arrival order
            r = waiting.pop(0)
            slot_of[r] = free_slots.pop(0)
            done_tok[r] = 0
            admitted[r] = n_admissions
            n_admissions += 1
        dec = [r for r in slot_of if done_tok[r] >= prompt[r]]
        chk = [r for r in slot_of if done_tok[r] < prompt[r]]
        chunk = [int(min(chunk_cap, prompt[r] - done_tok[r])) for r in chk]
        rows = dec + chk
        new = [1] * len(dec) + chunk
        k_new = torch.cat([hist_k[r][done_tok[r]:done_tok[r] + m] for r, m in zip(rows, new)])
        v_new = torch.cat([hist_v[r][done_tok[r]:done_tok[r] + m] for r, m in zip(rows, new)])
        q_dec = torch.randn(len(dec), Hq, D, generator=gen).to(torch.bfloat16)
        q_chk = torch.randn(sum(chunk), Hq, D, generator=gen).to(torch.bfloat16)
        st, d_res, c_res = drv.step([slot_of[r] for r in dec], [slot_of[r] for r in chk], chunk,
                                    k_new.cuda(), v_new.cuda(), q_dec.cuda(), q_chk.cuda(), scale)
        if st == pkv.PKV_ERR_NO_PAGES:
            # not enough pages for every row: preempt the youngest request
            # (its pages go back; it restarts later) and admit nobody until a
            # step fits again
            no_pages += 1
            victim = max(slot_of, key=lambda r: admitted[r])
            alloc.release(slot_of[victim])
            free_slots.append(slot_of.pop(victim))
            waiting.insert(0, victim)
            admit = False
            continue
        assert st == 0
        admit = True
        torch.cuda.synchronize()
        lens = [done_tok[r] + m for r, m in zip(rows, new)]
        if dec:
            ref, ref_lse = _reference(hist_k, hist_v, dec, lens[:len(dec)], q_dec, None, P_ref,
                                      Hkv, D, scale, "decode")
            compare(d_res[0], d_res[1], ref, ref_lse)
            checked += len(dec)
        if chk:
            cu_q = np.concatenate([[0], np.cumsum(chunk)])
            ref, ref_lse = _reference(hist_k, hist_v, chk, lens[len(dec):], q_chk, cu_q, P_ref,
                                      Hkv, D, scale, "prefill")
            compare(c_res[0], c_res[1], ref, ref_lse)
            checked += len(chk)
        for r, m in zip(rows, new):
            done_tok[r] += m
        # the allocator holds exactly the pages of the live lengths
        live = [done_tok[r] for r in slot_of]
        assert alloc.stats().pages_in_use == sum(pages_for(L, page_size) for L in live)
        for r in list(slot_of):
            if done_tok[r] >= total[r]:
                alloc.release(slot_of[r])
                free_slots.append(slot_of.pop(r))
    assert int(flags.item()) == 0
    assert alloc.stats().pages_in_use == 0
    assert checked >= n_req and steps > 10 and no_pages > 0
