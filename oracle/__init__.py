"""CPU oracle for attention over a paged KV cache (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path
and never imports it.  The arithmetic lives in ``oracle.c`` (plain fp64 C with
OpenMP over (sequence, kv head)); this module compiles it with gcc and wraps
it with ctypes over numpy arrays.

Functions and what they follow (pages on TensorRT-LLM):
* ``append``          paged KV store through the page table (concept page,
                      "PagedAttention 及 KV 快取管理"; "編譯期圖最佳化" page-table
                      lookup nodes for KV writes)
* ``decode``          textbook softmax(q K^T * scale) V over the gathered pages
                      ("執行時執行模型": attention reads the KV pages)
* ``prefill_chunk``   the same per query with a bottom-right causal limit
                      ("關鍵效能引數": context tokens in parallel over pages)
* ``decode_partial`` / ``merge``   split partials and their merge (the
                      split-KV decode formula; no counterpart on the pages)
* ``e4m3_*`` / ``fp8_quantize``    E4M3 codec from the format definition
                      (yololab.net guide, "FP8 與極致量化")
* ``int8_*``          symmetric INT8 codec (concept page, "關鍵機制"
                      quantisation bullet: INT8 KV cache)
* ``e2m1_*`` / ``nvfp4_*``   FP4 (E2M1) codec with E4M3 block scales per 16
                      values (solosoft post: FP4 quantisation needs
                      Blackwell; the block layout is a reading)

Every function is pinned by ``tests/test_oracle_*.py`` against brute force,
library special cases, closed forms and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")

KV_BF16 = 0
KV_E4M3 = 1
KV_INT8 = 2
KV_NVFP4 = 3

_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``_build/liboracle.so`` with gcc (-O2, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_D = ctypes.c_double
_F = ctypes.c_float


def _declare(L):
    L.oracle_num_threads.restype = _I
    L.oracle_set_num_threads.argtypes = [_I]
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = _D
    L.oracle_e4m3_encode.argtypes = [_F]
    L.oracle_e4m3_encode.restype = ctypes.c_uint8
    L.oracle_fp8_quotient.argtypes = [ctypes.c_uint16, _F]
    L.oracle_fp8_quotient.restype = _F
    L.oracle_e4m3_encode_array.argtypes = [_P, _P, _I64]
    L.oracle_e4m3_decode_array.argtypes = [_P, _P, _I64]
    L.oracle_fp8_quantize_array.argtypes = [_P, _P, _P, _I64]
    L.oracle_int8_encode.argtypes = [_F]
    L.oracle_int8_encode.restype = ctypes.c_int8
    L.oracle_int8_quantize_array.argtypes = [_P, _P, _P, _I64]
    L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_decode.restype = _D
    L.oracle_e2m1_encode.argtypes = [_F]
    L.oracle_e2m1_encode.restype = ctypes.c_uint8
    L.oracle_e2m1_encode_array.argtypes = [_P, _P, _I64]
    L.oracle_nvfp4_quantize_row.argtypes = [_P, _I64, _F, _P, _P]
    L.oracle_nvfp4_value.argtypes = [_P, _P, _F, _I64]
    L.oracle_nvfp4_value.restype = _D
    cache = [_P, _P, _P, _P, _I, _I, _I, _I, _I]
    L.oracle_append.argtypes = cache + [_P, _I, _P, _P, _I, _P, _P]
    L.oracle_append.restype = _I
    L.oracle_decode.argtypes = cache + [_P, _I, _P, _I, _P, _I, _D, _P, _I, _P, _P]
    L.oracle_decode.restype = _I
    L.oracle_prefill_chunk.argtypes = cache + [_P, _I, _P, _P, _I, _P, _I, _D, _P, _P]
    L.oracle_prefill_chunk.restype = _I
    L.oracle_decode_partial.argtypes = cache + [_P, _I, _P, _I, _P, _I, _D, _I, _I, _P, _P, _P]
    L.oracle_decode_partial.restype = _I
    L.oracle_merge.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P]
    L.oracle_merge.restype = _I


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops from now on."""
    lib().oracle_set_num_threads(int(n))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _check(status: int, what: str):
    if status != 0:
        raise RuntimeError(f"oracle {what} failed with status {status}")


# ------------------------------------------------------------------- codec
def e4m3_decode(codes) -> np.ndarray:
    codes = _c(codes, np.uint8)
    out = np.empty(codes.shape, np.float64)
    lib().oracle_e4m3_decode_array(_ptr(codes), _ptr(out), codes.size)
    return out


def e4m3_encode(y) -> np.ndarray:
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(y), _ptr(out), y.size)
    return out


def fp8_quantize(x_bits, scale) -> np.ndarray:
    """E4M3 codes of bf16 values (given as uint16 bits) divided by fp32 scales."""
    x_bits = _c(x_bits, np.uint16)
    scale = _c(np.broadcast_to(scale, x_bits.shape), np.float32)
    out = np.empty(x_bits.shape, np.uint8)
    lib().oracle_fp8_quantize_array(_ptr(x_bits), _ptr(scale), _ptr(out), x_bits.size)
    return out


def int8_encode(y) -> np.ndarray:
    """INT8 codes of fp32 values: nearest integer (ties to even) clamped to +-127, NaN -> 0."""
    y = _c(y, np.float32).reshape(-1)
    return np.array([lib().oracle_int8_encode(float(v)) for v in y], np.int8)


def int8_quantize(x_bits, scale) -> np.ndarray:
    """INT8 codes of bf16 values (given as uint16 bits) divided by fp32 scales."""
    x_bits = _c(x_bits, np.uint16)
    scale = _c(np.broadcast_to(scale, x_bits.shape), np.float32)
    out = np.empty(x_bits.shape, np.int8)
    lib().oracle_int8_quantize_array(_ptr(x_bits), _ptr(scale), _ptr(out), x_bits.size)
    return out


def e2m1_decode(codes) -> np.ndarray:
    """Values of E2M1 codes (low 4 bits), fp64."""
    return np.array([lib().oracle_e2m1_decode(int(c) & 0xF) for c in np.ravel(codes)],
                    np.float64).reshape(np.shape(codes))


def e2m1_encode(y) -> np.ndarray:
    """E2M1 codes of fp32 values: nearest, ties to even, saturating at +-6, NaN -> 0."""
    y = _c(y, np.float32)
    out = np.empty(y.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_ptr(y), _ptr(out), y.size)
    return out


def nvfp4_quantize(x_bits, scale):
    """NVFP4 codes of bf16 rows (uint16 bits ``[rows, n]``, n a multiple of 16)
    with one fp32 scale per row: ``(packed uint8 [rows, n/2], block scales
    uint8 [rows, n/16])``, the even element in the low nibble."""
    x_bits = _c(np.atleast_2d(x_bits), np.uint16)
    rows, n = x_bits.shape
    if n % 16:
        raise ValueError("row length must be a multiple of 16")
    scale = _c(np.broadcast_to(scale, (rows,)), np.float32)
    packed = np.empty((rows, n // 2), np.uint8)
    blocks = np.empty((rows, n // 16), np.uint8)
    for r in range(rows):
        lib().oracle_nvfp4_quantize_row(_ptr(x_bits[r]), n, float(scale[r]), _ptr(packed[r]),
                                        _ptr(blocks[r]))
    return packed, blocks


def nvfp4_dequantize(packed, blocks, scale) -> np.ndarray:
    """Stored values (fp64 ``[rows, n]``) of rows quantised by ``nvfp4_quantize``."""
    packed = _c(np.atleast_2d(packed), np.uint8)
    blocks = _c(np.atleast_2d(blocks), np.uint8)
    rows, n = packed.shape[0], packed.shape[1] * 2
    scale = _c(np.broadcast_to(scale, (rows,)), np.float32)
    out = np.empty((rows, n), np.float64)
    for r in range(rows):
        for i in range(n):
            out[r, i] = lib().oracle_nvfp4_value(_ptr(packed[r]), _ptr(blocks[r]),
                                                 float(scale[r]), i)
    return out


# ------------------------------------------------------------------- cache
class Cache:
    """A host KV pool image: K and V byte pools ``[pages][Hkv][P][D]`` plus scales.

    FP4 (``"nvfp4"``) pools hold the codes ``[pages][Hkv][P][D/2]`` (two per
    byte, the even element in the low nibble) followed by the E4M3 block
    scales ``[pages][Hkv][P][D/16]``.
    """

    def __init__(self, num_pages, page_size, num_kv_heads, head_dim, kv_dtype="bf16",
                 k_pool=None, v_pool=None, k_scale=None, v_scale=None):
        self.num_pages = int(num_pages)
        self.page_size = int(page_size)
        self.num_kv_heads = int(num_kv_heads)
        self.head_dim = int(head_dim)
        self.kv_dtype = kv_dtype
        self.code = {"bf16": KV_BF16, "e4m3": KV_E4M3, "int8": KV_INT8,
                     "nvfp4": KV_NVFP4}[kv_dtype]
        rows = self.num_pages * self.num_kv_heads * self.page_size
        if self.code == KV_NVFP4:
            nbytes = rows * (self.head_dim // 2 + self.head_dim // 16)
        else:
            nbytes = rows * self.head_dim * (2 if self.code == KV_BF16 else 1)
        self.k_pool = _c(k_pool, np.uint8) if k_pool is not None else np.zeros(nbytes, np.uint8)
        self.v_pool = _c(v_pool, np.uint8) if v_pool is not None else np.zeros(nbytes, np.uint8)
        assert self.k_pool.size == nbytes and self.v_pool.size == nbytes
        self.k_scale = None if k_scale is None else _c(k_scale, np.float32)
        self.v_scale = None if v_scale is None else _c(v_scale, np.float32)

    def _args(self):
        return (_ptr(self.k_pool), _ptr(self.v_pool), _ptr(self.k_scale), _ptr(self.v_scale),
                self.code, self.num_pages, self.page_size, self.num_kv_heads, self.head_dim)

    # ---------------------------------------------------------------- ops
    def append(self, page_table, seq_lens_before, cu_new, k_new_bits, v_new_bits):
        page_table = _c(page_table, np.int32)
        seq_lens_before = _c(seq_lens_before, np.int32)
        cu_new = _c(cu_new, np.int32)
        k_new_bits = _c(k_new_bits, np.uint16)
        v_new_bits = _c(v_new_bits, np.uint16)
        batch = seq_lens_before.shape[0]
        maxp = page_table.shape[1] if page_table.ndim == 2 else 1
        st = lib().oracle_append(*self._args(), _ptr(page_table), maxp, _ptr(seq_lens_before),
                                 _ptr(cu_new), batch, _ptr(k_new_bits), _ptr(v_new_bits))
        _check(st, "append")

    def decode(self, q_bits, page_table, seq_lens, softmax_scale, seq_ids=None):
        """fp64 (out [B,Hq,D], lse [B,Hq]); rows outside ``seq_ids`` are NaN."""
        q_bits = _c(q_bits, np.uint16)
        page_table = _c(page_table, np.int32)
        seq_lens = _c(seq_lens, np.int32)
        B, Hq, D = q_bits.shape
        out = np.full((B, Hq, D), np.nan)
        lse = np.full((B, Hq), np.nan)
        ids = None if seq_ids is None else _c(seq_ids, np.int32)
        st = lib().oracle_decode(*self._args(), _ptr(q_bits), Hq, _ptr(page_table),
                                 page_table.shape[1], _ptr(seq_lens), B, float(softmax_scale),
                                 _ptr(ids), 0 if ids is None else ids.size, _ptr(out), _ptr(lse))
        _check(st, "decode")
        return out, lse

    def prefill_chunk(self, q_bits, cu_q, page_table, seq_lens, softmax_scale):
        """fp64 (out [Tq,Hq,D], lse [Tq,Hq]) of causal chunk attention."""
        q_bits = _c(q_bits, np.uint16)
        cu_q = _c(cu_q, np.int32)
        page_table = _c(page_table, np.int32)
        seq_lens = _c(seq_lens, np.int32)
        T, Hq, D = q_bits.shape
        out = np.full((T, Hq, D), np.nan)
        lse = np.full((T, Hq), np.nan)
        st = lib().oracle_prefill_chunk(*self._args(), _ptr(q_bits), Hq, _ptr(cu_q),
                                        _ptr(page_table), page_table.shape[1], _ptr(seq_lens),
                                        seq_lens.shape[0], float(softmax_scale), _ptr(out),
                                        _ptr(lse))
        _check(st, "prefill_chunk")
        return out, lse

    def decode_partial(self, q_bits, page_table, seq_lens, softmax_scale, page_begin, page_end):
        q_bits = _c(q_bits, np.uint16)
        page_table = _c(page_table, np.int32)
        seq_lens = _c(seq_lens, np.int32)
        B, Hq, D = q_bits.shape
        acc = np.empty((B, Hq, D))
        m = np.empty((B, Hq))
        l = np.empty((B, Hq))
        st = lib().oracle_decode_partial(*self._args(), _ptr(q_bits), Hq, _ptr(page_table),
                                         page_table.shape[1], _ptr(seq_lens), B,
                                         float(softmax_scale), int(page_begin), int(page_end),
                                         _ptr(acc), _ptr(m), _ptr(l))
        _check(st, "decode_partial")
        return acc, m, l


def merge(acc, m, l):
    """Merge split partials: acc [n,rows,D], m/l [n,rows] -> (out [rows,D], lse [rows])."""
    acc = _c(acc, np.float64)
    m = _c(m, np.float64)
    l = _c(l, np.float64)
    n, rows, D = acc.shape
    out = np.empty((rows, D))
    lse = np.empty(rows)
    _check(lib().oracle_merge(n, rows, D, _ptr(acc), _ptr(m), _ptr(l), _ptr(out), _ptr(lse)),
           "merge")
    return out, lse


# -------------------------------------------------------- workload helpers
def bf16_bits(t) -> np.ndarray:
    """uint16 bit patterns of a bf16 torch tensor (no arithmetic)."""
    import torch

    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def cache_for(w, seq_ids=None, include_new=True) -> Cache:
    """Build this oracle's own pool for workload ``w`` by its own append.

    Every token of the chosen sequences (default: all) is stored through
    ``Cache.append`` with the workload's page table; all other bytes keep the
    NaN sentinel.  ``include_new=False`` stores only the context tokens.
    """
    from workloads import BF16_NAN_BITS, sentinel_byte

    seq_ids = range(w.batch) if seq_ids is None else list(seq_ids)
    if w.kv_dtype != "bf16":
        k_pool = np.full(w.pool_bytes(), sentinel_byte(w.kv_dtype), np.uint8)
        v_pool = np.full(w.pool_bytes(), sentinel_byte(w.kv_dtype), np.uint8)
        k_scale = np.ones((w.num_pages, w.num_kv_heads), np.float32)
        v_scale = np.ones((w.num_pages, w.num_kv_heads), np.float32)
    else:
        k_pool = np.full(w.pool_bytes() // 2, BF16_NAN_BITS, np.uint16).view(np.uint8)
        v_pool = np.full(w.pool_bytes() // 2, BF16_NAN_BITS, np.uint16).view(np.uint8)
        k_scale = v_scale = None
    c = Cache(w.num_pages, w.page_size, w.num_kv_heads, w.head_dim, w.kv_dtype,
              k_pool, v_pool, k_scale, v_scale)
    for b in seq_ids:
        k, v = w.kv_seq(b)
        if w.kv_dtype != "bf16":
            pages, ks, vs = w.kv_scales_for(b, k, v)
            c.k_scale[pages] = ks
            c.v_scale[pages] = vs
        n = int(w.ctx_lens[b]) + (int(w.new_lens[b]) if include_new else 0)
        c.append(w.page_table[b : b + 1], np.zeros(1, np.int32), np.array([0, n], np.int32),
                 bf16_bits(k[:n]), bf16_bits(v[:n]))
    return c
