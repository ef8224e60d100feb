"""Pins of the oracle's FP4 (NVFP4) KV pools, on CPU.

Pool layout (the reading the oracle documents): the codes of every row
[page][kv head][slot] (head_dim/2 bytes, even element in the low nibble),
then the E4M3 block scales of every row (head_dim/16 bytes).  Checked here:

* the append puts each token's codes and block scales where plain index
  arithmetic says, equal to the codec applied to that row with its
  (page, kv head) scale, and leaves every other byte at the 0x7F sentinel;
* context-then-new appends equal one append;
* decode and prefill equal the pure-Python brute force (its own E2M1 table,
  torch's E4M3) and fp64 torch SDPA on independently dequantised K/V;
* invariants: physical page permutation, chunk rows = truncated decodes.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import _brute

_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
_E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(
    torch.float64).numpy()


def _build(seed, ctx, new, P=4, Hq=4, Hkv=2, D=16, chunk_rows=(), slack=0.5, rng=None):
    return workloads.build("fp4", seed, ctx, new, page_size=P, num_q_heads=Hq,
                           num_kv_heads=Hkv, head_dim=D, kv_dtype="nvfp4", pool_slack=slack,
                           chunk_rows=chunk_rows, rng=rng)


def _q_bits(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return oracle.bf16_bits(torch.randn(*shape, generator=g).to(torch.bfloat16))


def _regions(w, pool):
    rows = w.num_pages * w.num_kv_heads * w.page_size
    D = w.head_dim
    codes = pool[:rows * D // 2].reshape(w.num_pages, w.num_kv_heads, w.page_size, D // 2)
    scales = pool[rows * D // 2:].reshape(w.num_pages, w.num_kv_heads, w.page_size, D // 16)
    return codes, scales


def _dequant(w, pool, scale):
    """fp64 [pages, Hkv, P, D] values of a whole FP4 pool, by plain indexing."""
    codes, blocks = _regions(w, pool)
    nib = np.empty(codes.shape[:-1] + (w.head_dim,), np.int64)
    nib[..., 0::2] = codes & 0xF
    nib[..., 1::2] = codes >> 4
    mag = _E2M1[nib & 7] * np.where(nib & 8, -1.0, 1.0)
    sb = np.repeat(_E4M3[blocks], 16, axis=-1)
    return mag * sb * scale.astype(np.float64)[:, :, None, None]


def test_append_layout_and_sentinels():
    w = _build(31, [0, 5, 9, 14], [1, 3, 1, 6], P=4, Hkv=2, D=32, slack=0.4)
    c = oracle.cache_for(w)
    written = np.zeros((w.num_pages, w.num_kv_heads, w.page_size), bool)
    for pool, which, sc in ((c.k_pool, 0, c.k_scale), (c.v_pool, 1, c.v_scale)):
        codes, blocks = _regions(w, pool)
        for b in range(w.batch):
            kv = w.kv_seq(b)[which]
            for t in range(int(w.lens_after[b])):
                page, slot = int(w.page_table[b, t // w.page_size]), t % w.page_size
                written[page, :, slot] = True
                for g in range(w.num_kv_heads):
                    want_c, want_b = oracle.nvfp4_quantize(oracle.bf16_bits(kv[t, g])[None],
                                                           sc[page, g])
                    assert np.array_equal(codes[page, g, slot], want_c[0])
                    assert np.array_equal(blocks[page, g, slot], want_b[0])
        assert np.all(codes[~written] == workloads.sentinel_byte("nvfp4"))
        assert np.all(blocks[~written] == workloads.sentinel_byte("nvfp4"))
    # unowned rows read as NaN (the block scale 0x7F is E4M3's NaN)
    vals = _dequant(w, c.k_pool, c.k_scale)
    assert np.all(np.isnan(vals[~written]))


def test_context_then_new_equals_one_append():
    w = _build(32, [3, 8, 0], [1, 5, 9], Hq=2, Hkv=1)
    whole = oracle.cache_for(w)
    step = oracle.cache_for(w, include_new=False)
    k_new, v_new = w.new_kv()
    step.append(w.page_table, w.ctx_lens, w.cu_new(), oracle.bf16_bits(k_new),
                oracle.bf16_bits(v_new))
    assert np.array_equal(whole.k_pool, step.k_pool)
    assert np.array_equal(whole.v_pool, step.v_pool)


def test_decode_matches_brute_force():
    w = _build(33, [0, 3, 4, 9], [1, 1, 1, 1])
    c = oracle.cache_for(w)
    q = _q_bits((4, 4, 16), 41)
    out, lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    bo, bl = _brute.decode(c, q, w.page_table, w.lens_after, w.softmax_scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


def test_prefill_matches_brute_force():
    w = _build(34, [0, 5, 2], [3, 4, 6], Hq=2, Hkv=1, chunk_rows=[0, 1, 2])
    c = oracle.cache_for(w)
    q = _q_bits((13, 2, 16), 42)
    cu = w.cu_q_chunks()
    out, lse = c.prefill_chunk(q, cu, w.page_table, w.lens_after, w.softmax_scale)
    bo, bl = _brute.prefill_chunk(c, q, cu, w.page_table, w.lens_after, w.softmax_scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("G", [1, 4])
def test_decode_matches_torch_sdpa(G):
    Hkv, D = 2, 32
    w = _build(35, [5, 40, 63, 64, 100], [1] * 5, P=16, Hq=Hkv * G, Hkv=Hkv, D=D)
    c = oracle.cache_for(w)
    q = _q_bits((5, Hkv * G, D), 43)
    out, lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    Kall, Vall = _dequant(w, c.k_pool, c.k_scale), _dequant(w, c.v_pool, c.v_scale)
    for b in range(5):
        n = int(w.lens_after[b])
        t = np.arange(n)
        pages, slots = w.page_table[b, t // w.page_size], t % w.page_size
        K = Kall[pages, :, slots, :].transpose(1, 0, 2)  # [Hkv, n, D]
        V = Vall[pages, :, slots, :].transpose(1, 0, 2)
        Kh, Vh = np.repeat(K, G, axis=0), np.repeat(V, G, axis=0)  # q head h reads h // G
        qf = (q[b].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qf[:, None, :])[None], torch.from_numpy(Kh)[None],
            torch.from_numpy(Vh)[None], scale=w.softmax_scale)[0, :, 0, :].numpy()
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_permuting_physical_pages_changes_nothing():
    ctx, new = [9, 0, 14], [1, 1, 1]
    wa = _build(36, ctx, new, slack=1.0)
    wb = _build(36, ctx, new, slack=1.0, rng=np.random.default_rng(77))
    assert not np.array_equal(wa.page_table, wb.page_table)
    ca, cb = oracle.cache_for(wa), oracle.cache_for(wb)
    q = _q_bits((3, 4, 16), 44)
    oa, la = ca.decode(q, wa.page_table, wa.lens_after, wa.softmax_scale)
    ob, lb = cb.decode(q, wb.page_table, wb.lens_after, wb.softmax_scale)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_chunk_rows_equal_truncated_decode():
    w = _build(37, [5, 0], [6, 1], chunk_rows=[0, 1])
    c = oracle.cache_for(w)
    T = int(w.new_lens.sum())
    q = _q_bits((T, 4, 16), 45)
    cu = w.cu_q_chunks()
    out, lse = c.prefill_chunk(q, cu, w.page_table, w.lens_after, w.softmax_scale)
    for ch in range(2):
        L, n = int(w.lens_after[ch]), int(w.new_lens[ch])
        for i in range(n):
            row = cu[ch] + i
            od, ld = c.decode(q[row:row + 1], w.page_table[ch:ch + 1], [L - n + i + 1],
                              w.softmax_scale)
            assert np.array_equal(out[row], od[0]) and np.array_equal(lse[row], ld[0])
