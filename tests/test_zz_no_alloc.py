"""Decode for callers that cannot allocate device memory (needs a GPU).

Some callers of this library are handed only input and output pointers and
may not call cudaMalloc or any allocator (a plugin inside a host framework
that owns all device memory, code running where allocation is forbidden).
``paged_decode_attention_noalloc`` serves them: its split partials live in a
16 MiB scratch array inside the library instead of a caller workspace.

This file checks, through the C ABI, that the allocation-free entry point
returns exactly what the workspace entry point returns at the same CTA count
(the same kernels over the same work split, so bit for bit) on two calls in
a row and on a following call with a different batch (the scratch keeps the
previous call's contents, which the new call must not read); that the
result matches the oracle within the parity bound; that once the first call
on the device has committed the array, further calls leave the device's
free memory unchanged; and that sizes beyond the scratch are rejected before
anything runs.  It is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu


def _noalloc(pkv, cache, q, table, lens, max_len, scale, num_ctas=0, out=None, lse=None):
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device) if lse is None else lse
    st = pkv.lib().paged_decode_attention_noalloc(
        ctypes.byref(cache.c_struct), ctypes.c_void_p(q.data_ptr()), q.shape[1],
        q.shape[1] // cache.num_kv_heads, ctypes.c_void_p(table.data_ptr()), table.shape[1],
        ctypes.c_void_p(lens.data_ptr()), q.shape[0], max_len, scale,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), num_ctas,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, lse


def _oracle_decode(w):
    c = oracle.cache_for(w)
    rows = w.decode_rows
    return c.decode(oracle.bf16_bits(w.q_decode()), w.page_table[rows], w.lens_after[rows],
                    w.softmax_scale)


def test_noalloc_decode_equals_workspace_decode_on_consecutive_calls():
    w = workloads.build("noalloc", 31, [100, 4000, 37, 2500, 900, 64, 3100, 1], [1] * 8,
                        page_size=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                        pool_slack=0.2)
    st = GpuState(w)
    st.append_step()
    pkv = st.pkv
    q, table, lens, max_len = st.decode_inputs()
    # the workspace entry point at the CTA count the automatic plan picks
    # (the same on both entry points: same device, same arguments)
    ref, ref_lse = pkv.paged_decode_attention(st.cache, q, table, lens, max_len, w.softmax_scale)
    for _ in range(2):  # two calls in a row share the scratch
        code, out, lse = _noalloc(pkv, st.cache, q, table, lens, max_len, w.softmax_scale)
        assert code == 0, pkv.pkv_status_string(code)
        torch.cuda.synchronize()
        assert torch.equal(out, ref) and torch.equal(lse, ref_lse)
    o_ref, l_ref = _oracle_decode(w)
    compare(out, lse, o_ref, l_ref)

    # a different batch next: the scratch still holds the previous partials
    w2 = workloads.build("noalloc2", 32, [700, 5, 1500], [1] * 3, page_size=128,
                         num_q_heads=16, num_kv_heads=2, head_dim=128, pool_slack=0.2)
    st2 = GpuState(w2)
    st2.append_step()
    q2, t2, l2, m2 = st2.decode_inputs()
    ref2, ref2_lse = pkv.paged_decode_attention(st2.cache, q2, t2, l2, m2, w2.softmax_scale,
                                                num_ctas=7)
    code, out2, lse2 = _noalloc(pkv, st2.cache, q2, t2, l2, m2, w2.softmax_scale, num_ctas=7)
    assert code == 0
    torch.cuda.synchronize()
    assert torch.equal(out2, ref2) and torch.equal(lse2, ref2_lse)
    assert int(st.flags.item()) == 0 and int(st2.flags.item()) == 0


def test_noalloc_calls_leave_free_device_memory_unchanged():
    w = workloads.build("noalloc3", 34, [300, 2000, 5], [1] * 3, page_size=64,
                        num_q_heads=32, num_kv_heads=8, head_dim=128, pool_slack=0.2)
    st = GpuState(w)
    st.append_step()
    pkv = st.pkv
    q, table, lens, max_len = st.decode_inputs()
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    # the first call on the device commits the scratch array (lazy module loading)
    code, _, _ = _noalloc(pkv, st.cache, q, table, lens, max_len, w.softmax_scale, out=out,
                          lse=lse)
    assert code == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        code, _, _ = _noalloc(pkv, st.cache, q, table, lens, max_len, w.softmax_scale, out=out,
                              lse=lse)
        assert code == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert int(st.flags.item()) == 0


def test_noalloc_rejects_requests_beyond_the_scratch():
    w = workloads.build("small", 33, [10], [1], page_size=64, num_q_heads=64, num_kv_heads=8,
                        head_dim=128)
    st = GpuState(w)
    pkv = st.pkv
    # 4096 sequences x 8 kv heads x 8 q heads of partials exceed 16 MiB
    need = pkv.paged_decode_workspace_bytes(4096, 64, 8, 128, 8192)
    assert need > pkv.NOALLOC_SCRATCH_BYTES
    # well-formed but fake (never dereferenced) pointers: the size check comes
    # after the argument checks and before anything is read or enqueued
    fake = 0x10000
    code = pkv.lib().paged_decode_attention_noalloc(
        ctypes.byref(st.cache.c_struct), fake, 64, 8, fake, 128, fake, 4096, 8192, 0.1, fake,
        None, 0, None)
    assert code == -11
    assert "16 MiB" in pkv.pkv_status_string(code)
