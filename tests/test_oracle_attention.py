"""Pins of the oracle's paged store and attention (CPU only).

What the pages fix (TensorRT-LLM concept page, "PagedAttention 及 KV 快取管理"
and "編譯期圖最佳化"): the page table is only a relabelling of storage, so the
result of attention over a paged cache must be that of textbook attention over
the same tokens laid out contiguously, whatever the physical placement.  The
oracle is checked against things other than itself:

* brute force in pure Python (``tests/_brute.py``) on tiny inputs,
* torch's ``scaled_dot_product_attention`` in fp64 (a library special case)
  over K/V gathered by plain numpy indexing,
* closed forms (one token, identical keys, zero scale, two tokens, lse),
* invariants (permuted pages, paged == contiguous, GQA == duplicated MHA,
  chunk of one query == decode, chunk row == truncated decode, merge of any
  page partition == unsplit).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import _brute


def _tiny(seed, ctx, new, P=4, Hq=4, Hkv=2, D=8, dtype="bf16", chunk_rows=(), slack=0.5,
          scale=None):
    w = workloads.build("tiny", seed, ctx, new, page_size=P, num_q_heads=Hq, num_kv_heads=Hkv,
                        head_dim=D, kv_dtype=dtype, pool_slack=slack, chunk_rows=chunk_rows,
                        softmax_scale=scale)
    return w, oracle.cache_for(w)


def _q_bits(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return oracle.bf16_bits(torch.randn(*shape, generator=g).to(torch.bfloat16))


def _contiguous_kv(w, c, b, n):
    """K, V fp64 [n, Hkv, D] of sequence b gathered by numpy indexing of the raw pools."""
    shape = (w.num_pages, w.num_kv_heads, w.page_size, w.head_dim)
    t = np.arange(n)
    pages = w.page_table[b, t // w.page_size]
    slots = t % w.page_size
    out = []
    for pool, scale in ((c.k_pool, c.k_scale), (c.v_pool, c.v_scale)):
        if w.kv_dtype == "e4m3":
            vals = torch.from_numpy(pool.copy()).view(torch.float8_e4m3fn).to(torch.float64)
            vals = vals.numpy().reshape(shape)
            x = vals[pages, :, slots, :] * scale[pages][:, :, None].astype(np.float64)
        elif w.kv_dtype == "int8":
            vals = pool.view(np.int8).astype(np.float64).reshape(shape)
            x = vals[pages, :, slots, :] * scale[pages][:, :, None].astype(np.float64)
        else:
            bits = pool.view(np.uint16).astype(np.uint32) << 16
            vals = bits.view(np.float32).astype(np.float64).reshape(shape)
            x = vals[pages, :, slots, :]
        out.append(x)
    return out


def _q_float(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sdpa(q, K, V, scale, mask=None):
    """fp64 torch SDPA: q [Hq, nq, D], K/V [Hq, n, D]."""
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        attn_mask=None if mask is None else torch.from_numpy(mask)[None, None], scale=scale)
    return o[0].numpy()


# ------------------------------------------------------------ brute force
@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
def test_decode_matches_brute_force(dtype):
    w, c = _tiny(1, [0, 3, 4, 9], [1, 1, 1, 1], dtype=dtype)
    q = _q_bits((4, 4, 8), 11)
    out, lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    bo, bl = _brute.decode(c, q, w.page_table, w.lens_after, w.softmax_scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
def test_prefill_matches_brute_force(dtype):
    w, c = _tiny(2, [0, 5, 2], [3, 4, 6], dtype=dtype, chunk_rows=[0, 1, 2], Hq=2, Hkv=1)
    q = _q_bits((13, 2, 8), 12)
    cu = w.cu_q_chunks()
    out, lse = c.prefill_chunk(q, cu, w.page_table, w.lens_after, w.softmax_scale)
    bo, bl = _brute.prefill_chunk(c, q, cu, w.page_table, w.lens_after, w.softmax_scale)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


# -------------------------------------------------- library special case
@pytest.mark.parametrize("dtype,G", [("bf16", 4), ("bf16", 1), ("e4m3", 8), ("int8", 8)])
def test_decode_matches_torch_sdpa(dtype, G):
    Hkv = 2
    w, c = _tiny(3, [5, 40, 63, 64, 100], [1] * 5, P=16, Hq=Hkv * G, Hkv=Hkv, D=32, dtype=dtype)
    q = _q_bits((5, Hkv * G, 32), 13)
    out, lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    for b in range(5):
        n = int(w.lens_after[b])
        K, V = _contiguous_kv(w, c, b, n)
        Kh = np.repeat(K.transpose(1, 0, 2), G, axis=0)  # q head h reads kv head h // G
        Vh = np.repeat(V.transpose(1, 0, 2), G, axis=0)
        ref = _sdpa(_q_float(q[b])[:, None, :], Kh, Vh, w.softmax_scale)[:, 0, :]
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)
        s = np.einsum("hd,htd->ht", _q_float(q[b]), Kh) * w.softmax_scale
        mx = s.max(axis=1, keepdims=True)
        ref_lse = (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True)))[:, 0]
        np.testing.assert_allclose(lse[b], ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
def test_prefill_matches_torch_sdpa_bottom_right_causal(dtype):
    Hkv, G, D = 2, 2, 16
    w, c = _tiny(4, [0, 7, 30], [9, 16, 5], P=8, Hq=Hkv * G, Hkv=Hkv, D=D, dtype=dtype,
                 chunk_rows=[0, 1, 2])
    T = int(w.new_lens.sum())
    q = _q_bits((T, Hkv * G, D), 14)
    cu = w.cu_q_chunks()
    out, lse = c.prefill_chunk(q, cu, w.page_table, w.lens_after, w.softmax_scale)
    for ch in range(3):
        L, n = int(w.lens_after[ch]), int(w.new_lens[ch])
        K, V = _contiguous_kv(w, c, ch, L)
        Kh = np.repeat(K.transpose(1, 0, 2), G, axis=0)
        Vh = np.repeat(V.transpose(1, 0, 2), G, axis=0)
        qq = _q_float(q[cu[ch]:cu[ch + 1]]).transpose(1, 0, 2)  # [Hq, n, D]
        pos = L - n + np.arange(n)
        mask = np.arange(L)[None, :] <= pos[:, None]
        ref = _sdpa(qq, Kh, Vh, w.softmax_scale, mask).transpose(1, 0, 2)
        np.testing.assert_allclose(out[cu[ch]:cu[ch + 1]], ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------- closed forms
def _cache_with_rows(K, V, P=4, scale=0.25, q=None, seed=0):
    """One sequence whose K/V rows are given (bf16-exact fp32 arrays [n, 1, D])."""
    n, _, D = K.shape
    w = workloads.build("closed", seed, [0], [n], page_size=P, num_q_heads=1, num_kv_heads=1,
                        head_dim=D, pool_slack=1.0, softmax_scale=scale)
    c = oracle.Cache(w.num_pages, P, 1, D)
    kb = oracle.bf16_bits(torch.from_numpy(K).to(torch.bfloat16))
    vb = oracle.bf16_bits(torch.from_numpy(V).to(torch.bfloat16))
    c.append(w.page_table, [0], [0, n], kb, vb)
    return w, c


def test_one_token_returns_its_v_row():
    w, c = _tiny(5, [0, 0], [1, 1], D=8)
    q = _q_bits((2, 4, 8), 15)
    out, lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    for b in range(2):
        K, V = _contiguous_kv(w, c, b, 1)
        for h in range(4):
            assert np.array_equal(out[b, h], V[0, h // 2])
            s = w.softmax_scale * float(_q_float(q[b, h]) @ K[0, h // 2])
            assert lse[b, h] == pytest.approx(s, abs=1e-14)


@pytest.mark.parametrize("scale", [0.0, 0.3])
def test_identical_keys_or_zero_scale_give_mean_of_v(scale):
    rng = np.random.default_rng(6)
    n, D = 11, 8
    krow = rng.standard_normal(D).astype(np.float32)
    K = np.repeat(krow[None, None], n, axis=0) if scale else rng.standard_normal((n, 1, D)).astype(np.float32)
    V = rng.standard_normal((n, 1, D)).astype(np.float32)
    w, c = _cache_with_rows(K, V, scale=scale)
    q = _q_bits((1, 1, D), 16)
    out, lse = c.decode(q, w.page_table, [n], scale)
    Vb = torch.from_numpy(V).to(torch.bfloat16).double().numpy()[:, 0]
    np.testing.assert_allclose(out[0, 0], Vb.mean(axis=0), rtol=0, atol=1e-14)
    Kb = torch.from_numpy(K).to(torch.bfloat16).double().numpy()[:, 0]
    s0 = scale * float(_q_float(q[0, 0]) @ Kb[0])
    if scale:
        assert lse[0, 0] == pytest.approx(s0 + math.log(n), abs=1e-12)
    else:
        assert lse[0, 0] == pytest.approx(math.log(n), abs=1e-14)


def test_two_tokens_sigmoid_form():
    rng = np.random.default_rng(7)
    D = 8
    K = rng.standard_normal((2, 1, D)).astype(np.float32)
    V = rng.standard_normal((2, 1, D)).astype(np.float32)
    w, c = _cache_with_rows(K, V, scale=0.7)
    q = _q_bits((1, 1, D), 17)
    out, lse = c.decode(q, w.page_table, [2], 0.7)
    Kb = torch.from_numpy(K).to(torch.bfloat16).double().numpy()[:, 0]
    Vb = torch.from_numpy(V).to(torch.bfloat16).double().numpy()[:, 0]
    qf = _q_float(q[0, 0])
    s1, s2 = 0.7 * qf @ Kb[0], 0.7 * qf @ Kb[1]
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    ref = sig(s1 - s2) * Vb[0] + sig(s2 - s1) * Vb[1]
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(math.exp(s1) + math.exp(s2)), abs=1e-13)


def test_empty_sequence_gives_zero_and_minus_inf():
    w, c = _tiny(8, [3], [1])
    q = _q_bits((1, 4, 8), 18)
    out, lse = c.decode(q, w.page_table, [0], w.softmax_scale)
    assert np.all(out == 0) and np.all(lse == -np.inf)


# -------------------------------------------------------------- invariants
def _same_tokens_other_placement(seed_a, seed_b, P_a, P_b, dtype="bf16"):
    """One set of token values stored under two page sizes/placements."""
    ctx, new = [9, 0, 14], [1, 1, 1]
    wa = workloads.build("a", seed_a, ctx, new, page_size=P_a, num_q_heads=4, num_kv_heads=2,
                         head_dim=8, kv_dtype=dtype, pool_slack=1.0)
    wb = workloads.build("a", seed_a, ctx, new, page_size=P_b, num_q_heads=4, num_kv_heads=2,
                         head_dim=8, kv_dtype=dtype, pool_slack=1.0,
                         rng=np.random.default_rng(seed_b))
    return wa, oracle.cache_for(wa), wb, oracle.cache_for(wb)


def test_permuting_physical_pages_changes_nothing():
    wa, ca, wb, cb = _same_tokens_other_placement(20, 99, 4, 4)
    assert not np.array_equal(wa.page_table, wb.page_table)
    q = _q_bits((3, 4, 8), 19)
    oa, la = ca.decode(q, wa.page_table, wa.lens_after, wa.softmax_scale)
    ob, lb = cb.decode(q, wb.page_table, wb.lens_after, wb.softmax_scale)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_paged_equals_contiguous():
    # P = 4 (several pages, permuted) against P = 64 >= L (one page per sequence,
    # identity table) holding the same token values.
    wa, ca, _, _ = _same_tokens_other_placement(21, 1, 4, 4)
    ctx, new = [9, 0, 14], [1, 1, 1]
    wc = workloads.build("a", 21, ctx, new, page_size=64, num_q_heads=4, num_kv_heads=2,
                         head_dim=8, pool_pages=3)
    wc.page_table[:, 0] = np.arange(3)
    cc = oracle.cache_for(wc)
    q = _q_bits((3, 4, 8), 20)
    oa, la = ca.decode(q, wa.page_table, wa.lens_after, wa.softmax_scale)
    oc, lc = cc.decode(q, wc.page_table, wc.lens_after, wc.softmax_scale)
    assert np.array_equal(oa, oc) and np.array_equal(la, lc)


def test_gqa_equals_mha_with_duplicated_kv_heads():
    G, Hkv, D, P = 4, 2, 8, 4
    w, c = _tiny(22, [6, 13], [1, 1], P=P, Hq=G * Hkv, Hkv=Hkv, D=D)
    q = _q_bits((2, G * Hkv, D), 21)
    og, lg = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    # MHA cache: kv head h holds a copy of GQA kv head h // G.
    shape = (w.num_pages, Hkv, P, D)
    mk = np.repeat(c.k_pool.view(np.uint16).reshape(shape), G, axis=1)
    mv = np.repeat(c.v_pool.view(np.uint16).reshape(shape), G, axis=1)
    cm = oracle.Cache(w.num_pages, P, G * Hkv, D, "bf16", mk.reshape(-1).view(np.uint8),
                      mv.reshape(-1).view(np.uint8))
    om, lm = cm.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    assert np.array_equal(og, om) and np.array_equal(lg, lm)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
def test_chunk_rows_equal_truncated_decode(dtype):
    w, c = _tiny(23, [5, 0], [6, 1], P=4, dtype=dtype, chunk_rows=[0, 1])
    T = int(w.new_lens.sum())
    q = _q_bits((T, 4, 8), 22)
    cu = w.cu_q_chunks()
    out, lse = c.prefill_chunk(q, cu, w.page_table, w.lens_after, w.softmax_scale)
    for ch in range(2):
        L, n = int(w.lens_after[ch]), int(w.new_lens[ch])
        for i in range(n):
            row = cu[ch] + i
            od, ld = c.decode(q[row:row + 1], w.page_table[ch:ch + 1], [L - n + i + 1],
                              w.softmax_scale)
            assert np.array_equal(out[row], od[0]) and np.array_equal(lse[row], ld[0])
    # the one-query chunk (sequence 1) is exactly a decode step


@pytest.mark.parametrize("cuts", [(1,), (1, 2), (2, 3), (0, 1, 3)])
def test_merge_of_any_page_partition_equals_unsplit(cuts):
    w, c = _tiny(24, [10, 3, 15], [1, 1, 1], P=4)
    q = _q_bits((3, 4, 8), 23)
    out, lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
    edges = [0, *cuts, w.max_pages_per_seq]
    parts = [c.decode_partial(q, w.page_table, w.lens_after, w.softmax_scale, a, b)
             for a, b in zip(edges[:-1], edges[1:])]
    acc = np.stack([p[0].reshape(-1, 8) for p in parts])
    m = np.stack([p[1].reshape(-1) for p in parts])
    l = np.stack([p[2].reshape(-1) for p in parts])
    mo, ml = oracle.merge(acc, m, l)
    np.testing.assert_allclose(mo.reshape(out.shape), out, rtol=0, atol=1e-14)
    np.testing.assert_allclose(ml.reshape(lse.shape), lse, rtol=0, atol=1e-13)


def test_bad_page_id_is_rejected():
    w, c = _tiny(25, [3], [1])
    bad = w.page_table.copy()
    bad[0, 0] = w.num_pages
    with pytest.raises(RuntimeError):
        c.decode(_q_bits((1, 4, 8), 1), bad, w.lens_after, w.softmax_scale)
