"""Every entry point rejects bad arguments on the host, before any CUDA call.

CPU only.  On a machine without a GPU a call that reached the CUDA runtime
would come back as PKV_ERR_CUDA (-8); getting the documented status instead
shows that the check ran first.  Pointers are fake, 16-byte aligned
addresses; none is ever dereferenced.
"""
import ctypes

import pytest

# status codes of include/paged_kv.h
OK, NULL, SHAPE, PAGE_SIZE, HEAD_DIM, GQA, DTYPE, WORKSPACE, CUDA, ALIGN = (
    0, -1, -2, -3, -4, -5, -6, -7, -8, -9)
A = 0x10000  # a fake aligned device address


@pytest.fixture(scope="module")
def pkv():
    import __graft_entry__

    __graft_entry__._builder().build()
    import paged_kv_cache_476_b200 as m

    return m


def _cache(pkv, **kw):
    c = pkv.PkvCache(A, A + 0x100000, None, None, 16, 64, 8, 128, pkv.PKV_KV_BF16, None)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _decode(pkv, fn="paged_decode_attention", c=None, q=A, Hq=32, G=4, table=A, maxp=4,
            lens=A, batch=2, max_len=100, scale=0.1, k_new=A, v_new=A, out=A, lse=None, ws=A,
            ws_bytes=1 << 30, ctas=0):
    L = pkv.lib()
    c = c or _cache(pkv)
    if fn == "paged_decode_attention_append":
        return L.paged_decode_attention_append(ctypes.byref(c), q, Hq, G, table, maxp, lens,
                                               batch, max_len, scale, k_new, v_new, out, lse, ws,
                                               ws_bytes, ctas, None)
    if fn == "paged_decode_attention_noalloc":
        return L.paged_decode_attention_noalloc(ctypes.byref(c), q, Hq, G, table, maxp, lens,
                                                batch, max_len, scale, out, lse, ctas, None)
    return L.paged_decode_attention(ctypes.byref(c), q, Hq, G, table, maxp, lens, batch,
                                    max_len, scale, out, lse, ws, ws_bytes, ctas, None)


DECODES = ["paged_decode_attention", "paged_decode_attention_append",
           "paged_decode_attention_noalloc"]


@pytest.mark.parametrize("fn", DECODES)
@pytest.mark.parametrize("kw,status", [
    ({"q": None}, NULL),
    ({"table": None}, NULL),
    ({"lens": None}, NULL),
    ({"out": None}, NULL),
    ({"q": A + 8}, ALIGN),
    ({"out": A + 4}, ALIGN),
    ({"batch": -1}, SHAPE),
    ({"maxp": 0}, SHAPE),
    ({"max_len": 64 * 4 + 1}, SHAPE),  # longer than the page table can map
    ({"scale": float("inf")}, SHAPE),
    ({"Hq": 24}, GQA),
    ({"G": 3, "Hq": 24}, GQA),
])
def test_decode_entry_points_reject(pkv, fn, kw, status):
    assert _decode(pkv, fn, **kw) == status


@pytest.mark.parametrize("fn", DECODES)
@pytest.mark.parametrize("field,value,status", [
    ("page_size", 32, PAGE_SIZE), ("head_dim", 96, HEAD_DIM), ("kv_dtype", 9, DTYPE),
    ("k_pool", None, NULL), ("v_pool", A + 8, ALIGN),
])
def test_decode_entry_points_reject_bad_cache(pkv, fn, field, value, status):
    assert _decode(pkv, fn, c=_cache(pkv, **{field: value})) == status


def test_one_byte_cache_without_scales(pkv):
    for fmt in (pkv.PKV_KV_FP8_E4M3, pkv.PKV_KV_INT8):
        assert _decode(pkv, c=_cache(pkv, kv_dtype=fmt)) == DTYPE


def test_fused_decode_needs_its_tokens(pkv):
    fn = "paged_decode_attention_append"
    assert _decode(pkv, fn, k_new=None) == NULL
    assert _decode(pkv, fn, v_new=None) == NULL
    assert _decode(pkv, fn, k_new=A + 2) == ALIGN
    assert _decode(pkv, fn, v_new=A + 8) == ALIGN


def test_empty_batch_is_a_no_op(pkv):
    for fn in DECODES:
        assert _decode(pkv, fn, batch=0, q=None, out=None, k_new=None, v_new=None) == OK


def _prefill(pkv, c=None, q=A, Hq=32, G=4, cu=A, table=A, maxp=4, lens=A, chunks=2, total=64,
             max_q=32, scale=0.1, out=A, lse=None):
    c = c or _cache(pkv)
    return pkv.lib().paged_prefill_chunk_attention(ctypes.byref(c), q, Hq, G, cu, table, maxp,
                                                   lens, chunks, total, max_q, scale, out, lse,
                                                   None)


@pytest.mark.parametrize("kw,status", [
    ({"q": None}, NULL), ({"cu": None}, NULL), ({"table": None}, NULL), ({"lens": None}, NULL),
    ({"out": None}, NULL), ({"q": A + 2}, ALIGN), ({"out": A + 8}, ALIGN),
    ({"chunks": -1}, SHAPE), ({"total": -5}, SHAPE), ({"maxp": 0}, SHAPE),
    ({"scale": float("nan")}, SHAPE), ({"Hq": 16}, GQA),
    ({"c": "page"}, PAGE_SIZE),
])
def test_prefill_rejects(pkv, kw, status):
    if kw.get("c") == "page":
        kw = {"c": _cache(pkv, page_size=48)}
    assert _prefill(pkv, **kw) == status


def test_prefill_without_queries_is_a_no_op(pkv):
    assert _prefill(pkv, chunks=0, q=None, out=None) == OK
    assert _prefill(pkv, total=0, q=None, out=None) == OK


@pytest.mark.parametrize("args,status", [
    ((A, A, 0, 4, 128, A, None), SHAPE),      # no parts
    ((A, A, 2, -1, 128, A, None), SHAPE),     # negative rows
    ((A, A, 2, 4, 96, A, None), HEAD_DIM),
    ((None, A, 2, 4, 128, A, None), NULL),
    ((A, None, 2, 4, 128, A, None), NULL),
    ((A, A, 2, 4, 128, None, None), NULL),
    ((A + 8, A, 2, 4, 128, A, None), ALIGN),
    ((A, A, 2, 4, 128, A + 8, None), ALIGN),
    ((None, None, 2, 0, 128, None, None), OK),  # no rows: nothing to do
])
def test_combine_rejects(pkv, args, status):
    assert pkv.lib().paged_attention_combine(*args, None) == status


def test_append_rejects_null_inputs(pkv):
    L = pkv.lib()
    c = _cache(pkv)
    # page_table, seq_lens_before, cu_new, k_new, v_new missing in turn
    full = [A, 4, A, A, 2, 8, A, A]
    for i in (0, 2, 3, 6, 7):
        args = list(full)
        args[i] = None
        st = L.paged_kv_append(ctypes.byref(c), *args, None)
        assert st == NULL, (i, st)


def test_bounded_wait_check_rejects_bad_arguments(pkv):
    L = pkv.lib()
    assert L.pkv_check_bounded_wait(None, 1000, None, None) == NULL
    assert L.pkv_check_bounded_wait(A, -1, None, None) == SHAPE
    assert L.pkv_check_bounded_wait(A, 2_000_000_001, None, None) == SHAPE


def test_page_table_span_must_fit_int32(pkv):
    # max_pages_per_seq * page_size above INT32_MAX: rejected, no int32 overflow
    L = pkv.lib()
    c = _cache(pkv)
    big = (1 << 31) // 64  # * 64 = 2^31
    assert _decode(pkv, c=c, maxp=big) == SHAPE
    assert _decode(pkv, fn="paged_decode_attention_noalloc", c=c, maxp=big) == SHAPE
    assert L.paged_kv_append(ctypes.byref(c), A, big, A, A, 2, 5, A, A, None) == SHAPE
    assert L.paged_prefill_chunk_attention(ctypes.byref(c), A, 32, 4, A, A, big, A, 2, 10, 5,
                                           0.1, A, None, None) == SHAPE
