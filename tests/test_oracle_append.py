"""Pins of the oracle's paged KV store (CPU only).

TensorRT-LLM concept page, "PagedAttention 及 KV 快取管理" / "編譯期圖最佳化":
a token's K/V is written to the physical page the page table names for its
logical position.  Checked here by reading the pool back with plain numpy
indexing (gather returns the input bits; every other byte keeps its sentinel)
and, for E4M3, against torch's float8 cast of the IEEE fp32 quotient.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def _written_mask(w, n_of):
    """Boolean [pages, Hkv, P] of slots that hold a token."""
    m = np.zeros((w.num_pages, w.num_kv_heads, w.page_size), bool)
    for b in range(w.batch):
        t = np.arange(n_of(b))
        m[w.page_table[b, t // w.page_size], :, t % w.page_size] = True
    return m


@pytest.mark.parametrize("P", [4, 64])
def test_bf16_append_stores_bits_through_page_table(P):
    w = workloads.build("a", 3, [0, 5, 63, 64, 130], [1, 2, 1, 3, 1], page_size=P,
                        num_q_heads=4, num_kv_heads=2, head_dim=16, pool_slack=0.3)
    c = oracle.cache_for(w)
    shape = (w.num_pages, w.num_kv_heads, w.page_size, w.head_dim)
    kp = c.k_pool.view(np.uint16).reshape(shape)
    vp = c.v_pool.view(np.uint16).reshape(shape)
    for b in range(w.batch):
        k, v = w.kv_seq(b)
        t = np.arange(int(w.lens_after[b]))
        got_k = kp[w.page_table[b, t // P], :, t % P, :]
        got_v = vp[w.page_table[b, t // P], :, t % P, :]
        assert np.array_equal(got_k, oracle.bf16_bits(k))
        assert np.array_equal(got_v, oracle.bf16_bits(v))
    untouched = ~_written_mask(w, lambda b: int(w.lens_after[b]))
    assert np.all(kp[untouched] == workloads.BF16_NAN_BITS)
    assert np.all(vp[untouched] == workloads.BF16_NAN_BITS)


def test_e4m3_append_matches_library_quantisation():
    w = workloads.build("a", 4, [0, 17, 64], [1, 1, 65], page_size=16, num_q_heads=8,
                        num_kv_heads=2, head_dim=32, kv_dtype="e4m3", pool_slack=0.2)
    c = oracle.cache_for(w)
    shape = (w.num_pages, w.num_kv_heads, w.page_size, w.head_dim)
    kp = c.k_pool.reshape(shape)
    vp = c.v_pool.reshape(shape)
    P = w.page_size
    for b in range(w.batch):
        k, v = w.kv_seq(b)
        t = np.arange(int(w.lens_after[b]))
        pages = w.page_table[b, t // P]
        for pool, src, sc in ((kp, k, c.k_scale), (vp, v, c.v_scale)):
            s = sc[pages][:, :, None]  # [n, Hkv, 1]
            y = (src.float().numpy() / s).astype(np.float32)
            ref = torch.from_numpy(np.clip(y, -448, 448)).to(torch.float8_e4m3fn)
            ref = ref.view(torch.uint8).numpy()
            got = pool[pages, :, t % P, :]
            nz = (ref & 0x7F) != 0
            assert np.array_equal(got[nz], ref[nz])
            assert np.all((got[~nz] & 0x7F) == 0)
            # absmax / 448 scales: the largest magnitude of each page lands on 448
            assert np.abs(y).max() <= 448.0 * (1 + 2**-20)
    untouched = ~_written_mask(w, lambda b: int(w.lens_after[b]))
    assert np.all(kp[untouched] == workloads.E4M3_NAN_CODE)
    assert np.all(vp[untouched] == workloads.E4M3_NAN_CODE)


def test_int8_append_matches_library_rounding():
    w = workloads.build("a", 7, [0, 17, 64], [1, 1, 65], page_size=16, num_q_heads=8,
                        num_kv_heads=2, head_dim=32, kv_dtype="int8", pool_slack=0.2)
    c = oracle.cache_for(w)
    shape = (w.num_pages, w.num_kv_heads, w.page_size, w.head_dim)
    kp = c.k_pool.view(np.int8).reshape(shape)
    vp = c.v_pool.view(np.int8).reshape(shape)
    P = w.page_size
    for b in range(w.batch):
        k, v = w.kv_seq(b)
        t = np.arange(int(w.lens_after[b]))
        pages = w.page_table[b, t // P]
        for pool, src, sc in ((kp, k, c.k_scale), (vp, v, c.v_scale)):
            s = sc[pages][:, :, None]  # [n, Hkv, 1]
            y = (src.float().numpy() / s).astype(np.float32)  # IEEE fp32 quotient
            ref = np.clip(np.rint(y), -127, 127).astype(np.int8)  # ties to even
            assert np.array_equal(pool[pages, :, t % P, :], ref)
            # absmax / 127 scales: the largest magnitude of each page lands on 127
            assert np.abs(y).max() <= 127.0 * (1 + 2**-20)
    untouched = ~_written_mask(w, lambda b: int(w.lens_after[b]))
    assert np.all(c.k_pool.reshape(shape)[untouched] == workloads.INT8_UNOWNED)
    assert np.all(c.v_pool.reshape(shape)[untouched] == workloads.INT8_UNOWNED)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
def test_context_then_new_equals_one_append(dtype):
    w = workloads.build("a", 5, [3, 8, 0], [1, 5, 9], page_size=4, num_q_heads=2,
                        num_kv_heads=1, head_dim=8, kv_dtype=dtype, pool_slack=0.5)
    whole = oracle.cache_for(w)
    step = oracle.cache_for(w, include_new=False)
    k_new, v_new = w.new_kv()
    step.append(w.page_table, w.ctx_lens, w.cu_new(), oracle.bf16_bits(k_new),
                oracle.bf16_bits(v_new))
    assert np.array_equal(whole.k_pool, step.k_pool)
    assert np.array_equal(whole.v_pool, step.v_pool)


def test_append_past_the_page_table_is_rejected():
    w = workloads.build("a", 6, [4], [1], page_size=4, num_q_heads=1, num_kv_heads=1,
                        head_dim=8)
    c = oracle.cache_for(w)
    k = oracle.bf16_bits(torch.zeros(1, 1, 8, dtype=torch.bfloat16))
    with pytest.raises(RuntimeError):
        c.append(w.page_table, [8], [0, 1], k, k)  # position 8 needs a third page
