"""The C-ABI library builds, loads and exports every symbol its header declares.

CPU only: no call here reaches a kernel.  Argument errors are returned by the
host-side validation before any CUDA call, so they can be checked without a
GPU, and the decode plan is pure host arithmetic.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(os.path.join(ROOT, "include", h) for h in os.listdir(os.path.join(ROOT, "include"))
                 if h.endswith(".h"))


@pytest.fixture(scope="module")
def pkv():
    import __graft_entry__

    __graft_entry__._builder().build()
    import paged_kv_cache_476_b200 as m

    return m


def _declared_functions():
    text = "\n".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("paged_kv_append", "paged_decode_attention", "paged_prefill_chunk_attention"):
        assert n in names


def test_library_exports_every_declared_symbol(pkv):
    lib = ctypes.CDLL(pkv.LIB_PATH)
    declared = _declared_functions()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(declared) == set(pkv.EXPORTED)


def test_status_strings_and_version(pkv):
    assert pkv.pkv_status_string(0) == "ok"
    for s in range(-12, 0):
        assert pkv.pkv_status_string(s) != "unknown status"
    assert pkv.lib().pkv_abi_version() >> 16 == 1


def _cache(pkv, **kw):
    c = pkv.PkvCache(0x1000, 0x2000, None, None, 16, 64, 8, 128, pkv.PKV_KV_BF16, None)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status", [
    ("page_size", 32, -3),
    ("head_dim", 96, -4),
    ("kv_dtype", 7, -6),
    ("num_pages", 0, -2),
    ("k_pool", None, -1),
    ("k_pool", 0x1008, -9),
])
def test_append_rejects_bad_cache_before_any_cuda_call(pkv, field, value, status):
    c = _cache(pkv, **{field: value})
    st = pkv.lib().paged_kv_append(ctypes.byref(c), None, 1, None, None, 1, 1, None, None, None)
    assert st == status


def test_e4m3_cache_needs_scales(pkv):
    c = _cache(pkv, kv_dtype=pkv.PKV_KV_FP8_E4M3)
    st = pkv.lib().paged_kv_append(ctypes.byref(c), None, 1, None, None, 1, 1, None, None, None)
    assert st == -6


def test_decode_rejects_bad_group_before_any_cuda_call(pkv):
    c = _cache(pkv)
    L = pkv.lib()
    # 8 kv heads * group 4 != 24 q heads
    st = L.paged_decode_attention(ctypes.byref(c), None, 24, 4, None, 1, None, 1, 64, 0.1, None,
                                  None, None, 0, 0, None)
    assert st == -5
    st = L.paged_decode_attention(ctypes.byref(c), None, 24, 3, None, 1, None, 1, 64, 0.1, None,
                                  None, None, 0, 0, None)
    assert st == -5


def test_prefill_rejects_bad_cache(pkv):
    c = _cache(pkv, page_size=16)
    st = pkv.lib().paged_prefill_chunk_attention(ctypes.byref(c), None, 32, 4, None, None, 1,
                                                 None, 1, 1, 1, 0.1, None, None, None)
    assert st == -3


def test_decode_plan_fills_the_machine_and_caps_at_the_work(pkv):
    # automatic: SMs x resident CTAs
    assert pkv.paged_decode_plan(64, 8, 4097, 148, 0, 1) == 148
    assert pkv.paged_decode_plan(64, 8, 4097, 148, 0, 2) == 296
    # never more CTAs than 64-token tiles of the largest batch
    assert pkv.paged_decode_plan(4, 8, 131, 148, 0, 2) == 4 * 8 * 3
    assert pkv.paged_decode_plan(1, 1, 1, 148, 0, 2) == 1
    # forced count
    assert pkv.paged_decode_plan(64, 8, 4097, 148, 13, 1) == 13
    # batch 0 still plans one (idle) CTA
    assert pkv.paged_decode_plan(0, 8, 0, 148, 0, 1) == 1
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_decode_plan(-1, 8, 10, 148)


def test_package_has_no_cpu_fallback():
    """The product path must not import or run the oracle."""
    pkg = os.path.join(ROOT, "paged_kv_cache_476_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
