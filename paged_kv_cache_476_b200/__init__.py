"""Attention over a paged KV cache on B200: Python binding of ``libpagedkv.so``.

A thin ctypes layer over the C ABI in ``include/paged_kv.h``: it checks and
marshals torch tensors (device memory, streams) into plain pointers and sizes
and calls the library.  Every step of the computation runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback.  If the library is missing
or cannot load, importing this package raises.

Entry points (same names as the C ABI):
    paged_kv_append                 paged store of new tokens' K/V (bf16, E4M3, INT8, FP4)
    paged_decode_attention          split-KV decode, persistent and balanced
    paged_prefill_chunk_attention   causal prefill chunks on tcgen05
    paged_decode_workspace_bytes, paged_decode_plan, pkv_status_string
    PageAllocator                   host page allocator + in-flight step planner
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpagedkv.so")

PKV_KV_BF16 = 0
PKV_KV_FP8_E4M3 = 1
PKV_KV_INT8 = 2
PKV_KV_NVFP4 = 3
_KV_CODES = {"bf16": PKV_KV_BF16, "e4m3": PKV_KV_FP8_E4M3, "int8": PKV_KV_INT8,
             "nvfp4": PKV_KV_NVFP4}
PKV_FLAG_BAD_PAGE = 0x1
PKV_FLAG_BAD_LENGTH = 0x2
PKV_FLAG_TIMEOUT = 0x4
PKV_FLAG_BAD_SCALE = 0x8
PKV_ERR_NO_PAGES = -12

# Every symbol include/paged_kv.h declares.
EXPORTED = (
    "paged_kv_append",
    "paged_decode_plan",
    "paged_decode_workspace_bytes",
    "paged_decode_attention",
    "paged_prefill_chunk_attention",
    "pkv_status_string",
    "pkv_abi_version",
    "paged_decode_attention_noalloc",
    "paged_attention_combine",
    "paged_decode_attention_append",
    "pkv_check_bounded_wait",
    # include/paged_kv_runtime.h: host page allocator and step planner
    "pkv_allocator_create",
    "pkv_allocator_destroy",
    "pkv_allocator_grow",
    "pkv_allocator_release",
    "pkv_allocator_seq_len",
    "pkv_allocator_table",
    "pkv_allocator_stats",
    "pkv_allocator_free_pages",
    "pkv_step_plan",
)

# Size of the library's static decode scratch (see paged_decode_attention_noalloc).
NOALLOC_SCRATCH_BYTES = 16 << 20


class PkvCache(ctypes.Structure):
    """Mirror of ``struct pkv_cache``."""

    _fields_ = [
        ("k_pool", ctypes.c_void_p),
        ("v_pool", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("num_pages", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32),
        ("error_flags", ctypes.c_void_p),
    ]


class AllocStats(ctypes.Structure):
    """Mirror of ``struct pkv_alloc_stats``."""

    _fields_ = [
        ("num_pages", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_seqs", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("pages_in_use", ctypes.c_int32),
        ("peak_pages_in_use", ctypes.c_int32),
        ("live_seqs", ctypes.c_int32),
        ("tokens_cached", ctypes.c_int64),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python paged_kv_cache_476_b200/build.py` "
            "(there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    missing = [n for n in EXPORTED if not hasattr(lib, n)]
    if missing:
        raise ImportError(f"{LIB_PATH} is stale (missing {missing}): rebuild it with "
                          "`python paged_kv_cache_476_b200/build.py`")
    P, I32, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    cp = ctypes.POINTER(PkvCache)
    lib.paged_kv_append.argtypes = [cp, P, I32, P, P, I32, I32, P, P, P]
    lib.paged_kv_append.restype = ctypes.c_int
    lib.paged_decode_plan.argtypes = [I32, I32, I32, I32, I32, I32, ctypes.POINTER(I32)]
    lib.paged_decode_plan.restype = ctypes.c_int
    lib.paged_decode_workspace_bytes.argtypes = [I32, I32, I32, I32, I32, I32]
    lib.paged_decode_workspace_bytes.restype = SZ
    lib.paged_decode_attention.argtypes = [cp, P, I32, I32, P, I32, P, I32, I32, F, P, P, P, SZ,
                                           I32, P]
    lib.paged_decode_attention.restype = ctypes.c_int
    lib.paged_decode_attention_append.argtypes = [cp, P, I32, I32, P, I32, P, I32, I32, F, P, P,
                                                  P, P, P, SZ, I32, P]
    lib.paged_decode_attention_append.restype = ctypes.c_int
    lib.paged_prefill_chunk_attention.argtypes = [cp, P, I32, I32, P, P, I32, P, I32, I32, I32,
                                                  F, P, P, P]
    lib.paged_prefill_chunk_attention.restype = ctypes.c_int
    lib.paged_decode_attention_noalloc.argtypes = [cp, P, I32, I32, P, I32, P, I32, I32, F, P, P,
                                                   I32, P]
    lib.paged_decode_attention_noalloc.restype = ctypes.c_int
    lib.paged_attention_combine.argtypes = [P, P, I32, I32, I32, P, P, P]
    lib.paged_attention_combine.restype = ctypes.c_int
    lib.pkv_check_bounded_wait.argtypes = [P, ctypes.c_int64, P, P]
    lib.pkv_check_bounded_wait.restype = ctypes.c_int
    lib.pkv_status_string.argtypes = [ctypes.c_int]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_abi_version.restype = ctypes.c_int
    ap = ctypes.c_void_p
    pi = ctypes.POINTER(I32)
    lib.pkv_allocator_create.argtypes = [I32, I32, I32, I32, pi, ctypes.POINTER(ap)]
    lib.pkv_allocator_destroy.argtypes = [ap]
    lib.pkv_allocator_destroy.restype = None
    lib.pkv_allocator_grow.argtypes = [ap, I32, I32]
    lib.pkv_allocator_release.argtypes = [ap, I32]
    lib.pkv_allocator_seq_len.argtypes = [ap, I32, pi]
    lib.pkv_allocator_table.argtypes = [ap]
    lib.pkv_allocator_table.restype = pi
    lib.pkv_allocator_stats.argtypes = [ap, ctypes.POINTER(AllocStats)]
    lib.pkv_allocator_free_pages.argtypes = [ap, pi, I32, pi]
    lib.pkv_step_plan.argtypes = [ap, pi, pi, I32, pi, pi, pi, pi]
    for n in ("pkv_allocator_create", "pkv_allocator_grow", "pkv_allocator_release",
              "pkv_allocator_seq_len", "pkv_allocator_stats", "pkv_allocator_free_pages",
              "pkv_step_plan"):
        getattr(lib, n).restype = ctypes.c_int
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def pkv_status_string(status: int) -> str:
    return _lib.pkv_status_string(int(status)).decode()


class PagedKVError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what} failed: {pkv_status_string(status)} (status {status})")
        self.status = status


def _check(what: str, status: int):
    if status != 0:
        raise PagedKVError(what, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(name: str, t: torch.Tensor, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return t


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def nvfp4_pool_bytes(num_pages: int, num_kv_heads: int, page_size: int, head_dim: int) -> int:
    """Bytes of one FP4 pool: every row's E2M1 codes (head_dim/2 bytes), then
    every row's E4M3 block scales (head_dim/16 bytes)."""
    rows = num_pages * num_kv_heads * page_size
    return rows * (head_dim // 2 + head_dim // 16)


class PagedKVCache:
    """Caller-owned paged KV pool: K and V ``[num_pages, Hkv, page_size, head_dim]``.

    ``kv_dtype`` is ``"bf16"`` (torch.bfloat16 pools), ``"e4m3"`` (uint8 or
    float8_e4m3fn pools), ``"int8"`` (int8 or uint8 pools) or ``"nvfp4"``
    (FP4: flat uint8 pools of ``nvfp4_pool_bytes(...)`` bytes, codes then
    block scales, with ``geometry=(num_pages, Hkv, page_size, head_dim)``).
    The quantised formats take fp32 ``k_scale``/``v_scale`` ``[num_pages, Hkv]``.
    ``error_flags`` is an optional int32 device scalar that kernels OR
    ``PKV_FLAG_*`` bits into.
    """

    def __init__(self, k_pool, v_pool, kv_dtype="bf16", k_scale=None, v_scale=None,
                 error_flags=None, geometry=None):
        if kv_dtype not in _KV_CODES:
            raise ValueError("kv_dtype must be 'bf16', 'e4m3', 'int8' or 'nvfp4'")
        if kv_dtype == "nvfp4":
            if geometry is None or len(geometry) != 4:
                raise ValueError("FP4 pools need geometry=(num_pages, Hkv, page_size, head_dim)")
            _dev("k_pool", k_pool, torch.uint8, 1)
            _dev("v_pool", v_pool, torch.uint8, 1)
            need = nvfp4_pool_bytes(*geometry)
            if k_pool.numel() != need or v_pool.numel() != need:
                raise ValueError(f"FP4 pools of this geometry hold {need} bytes")
            shape = tuple(int(x) for x in geometry)
        else:
            dt = {"bf16": torch.bfloat16, "e4m3": (torch.uint8, torch.float8_e4m3fn),
                  "int8": (torch.int8, torch.uint8)}[kv_dtype]
            _dev("k_pool", k_pool, dt, 4)
            _dev("v_pool", v_pool, dt, 4)
            if k_pool.shape != v_pool.shape:
                raise ValueError("k_pool and v_pool shapes differ")
            shape = tuple(k_pool.shape)
        if kv_dtype != "bf16":
            if k_scale is None or v_scale is None:
                raise ValueError("quantised pools need k_scale and v_scale")
            _dev("k_scale", k_scale, torch.float32, 2)
            _dev("v_scale", v_scale, torch.float32, 2)
        if error_flags is not None:
            _dev("error_flags", error_flags, torch.int32)
        self.k_pool, self.v_pool = k_pool, v_pool
        self.k_scale, self.v_scale = k_scale, v_scale
        self.error_flags = error_flags
        self.kv_dtype = kv_dtype
        self.num_pages, self.num_kv_heads, self.page_size, self.head_dim = shape
        self._c = PkvCache(k_pool.data_ptr(), v_pool.data_ptr(),
                           None if k_scale is None else k_scale.data_ptr(),
                           None if v_scale is None else v_scale.data_ptr(),
                           self.num_pages, self.page_size, self.num_kv_heads, self.head_dim,
                           _KV_CODES[kv_dtype],
                           None if error_flags is None else error_flags.data_ptr())

    @property
    def c_struct(self) -> PkvCache:
        return self._c


def paged_kv_append(cache: PagedKVCache, page_table, seq_lens_before, cu_new_tokens, k_new,
                    v_new, total_new_tokens: Optional[int] = None, stream=None) -> None:
    """Store new tokens' K/V (bf16 ``[T, Hkv, D]``) into their pages."""
    _dev("page_table", page_table, torch.int32, 2)
    _dev("seq_lens_before", seq_lens_before, torch.int32, 1)
    _dev("cu_new_tokens", cu_new_tokens, torch.int32, 1)
    _dev("k_new", k_new, torch.bfloat16, 3)
    _dev("v_new", v_new, torch.bfloat16, 3)
    T = k_new.shape[0] if total_new_tokens is None else int(total_new_tokens)
    st = _lib.paged_kv_append(ctypes.byref(cache.c_struct), _ptr(page_table),
                              page_table.shape[1], _ptr(seq_lens_before), _ptr(cu_new_tokens),
                              seq_lens_before.shape[0], T, _ptr(k_new), _ptr(v_new),
                              _stream(stream))
    _check("paged_kv_append", st)


def paged_decode_plan(batch, num_kv_heads, max_seq_len, num_sms, num_ctas=0, ctas_per_sm=1):
    out = ctypes.c_int32(0)
    _check("paged_decode_plan", _lib.paged_decode_plan(batch, num_kv_heads, max_seq_len,
                                                       num_sms, num_ctas, ctas_per_sm,
                                                       ctypes.byref(out)))
    return out.value


def paged_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                 num_ctas=0) -> int:
    n = _lib.paged_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim,
                                          max_seq_len, num_ctas)
    if n == 0:
        raise PagedKVError("paged_decode_workspace_bytes", -2)
    return int(n)


def decode_workspace(cache: PagedKVCache, batch, num_q_heads, max_seq_len, num_ctas=0):
    """A zero-filled workspace tensor for paged_decode_attention."""
    n = paged_decode_workspace_bytes(batch, num_q_heads, cache.num_kv_heads, cache.head_dim,
                                     max_seq_len, num_ctas)
    return torch.zeros(n, dtype=torch.uint8, device=cache.k_pool.device)


def paged_decode_attention(cache: PagedKVCache, q, page_table, seq_lens, max_seq_len: int,
                           softmax_scale: Optional[float] = None, out=None, lse=None,
                           workspace=None, num_ctas: int = 0, want_lse: bool = True,
                           stream=None):
    """Decode attention of ``q`` bf16 ``[B, Hq, D]`` over the paged cache.

    Returns ``(out bf16 [B, Hq, D], lse fp32 [B, Hq] or None)``.
    """
    _dev("q", q, torch.bfloat16, 3)
    _dev("page_table", page_table, torch.int32, 2)
    _dev("seq_lens", seq_lens, torch.int32, 1)
    B, Hq, D = q.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(cache, B, Hq, max_seq_len, num_ctas)
    st = _lib.paged_decode_attention(
        ctypes.byref(cache.c_struct), _ptr(q), Hq, Hq // cache.num_kv_heads, _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, int(max_seq_len), float(softmax_scale),
        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), int(num_ctas), _stream(stream))
    _check("paged_decode_attention", st)
    return out, lse


def paged_decode_attention_append(cache: PagedKVCache, q, page_table, seq_lens, max_seq_len: int,
                                  k_new, v_new, softmax_scale: Optional[float] = None, out=None,
                                  lse=None, workspace=None, num_ctas: int = 0,
                                  want_lse: bool = True, stream=None):
    """A decode step with the append fused in.

    ``k_new``/``v_new`` bf16 ``[B, Hkv, D]`` hold each sequence's new token,
    stored at position ``seq_lens[b] - 1`` (``seq_lens`` counts it) by the
    same launch that then attends over all ``seq_lens[b]`` tokens.  Equal to
    ``paged_kv_append`` of one token per sequence followed by
    ``paged_decode_attention``.  Returns ``(out, lse)`` like the latter.
    """
    _dev("q", q, torch.bfloat16, 3)
    _dev("page_table", page_table, torch.int32, 2)
    _dev("seq_lens", seq_lens, torch.int32, 1)
    _dev("k_new", k_new, torch.bfloat16, 3)
    _dev("v_new", v_new, torch.bfloat16, 3)
    B, Hq, D = q.shape
    if tuple(k_new.shape) != (B, cache.num_kv_heads, D) or k_new.shape != v_new.shape:
        raise ValueError("k_new and v_new must be [batch, num_kv_heads, head_dim]")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(cache, B, Hq, max_seq_len, num_ctas)
    st = _lib.paged_decode_attention_append(
        ctypes.byref(cache.c_struct), _ptr(q), Hq, Hq // cache.num_kv_heads, _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, int(max_seq_len), float(softmax_scale),
        _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        int(num_ctas), _stream(stream))
    _check("paged_decode_attention_append", st)
    return out, lse


def paged_prefill_chunk_attention(cache: PagedKVCache, q, cu_q_lens, page_table, seq_lens,
                                  max_q_len: int, softmax_scale: Optional[float] = None,
                                  out=None, lse=None, want_lse: bool = True, stream=None):
    """Causal chunk attention of packed ``q`` bf16 ``[Tq, Hq, D]`` over the paged cache."""
    _dev("q", q, torch.bfloat16, 3)
    _dev("cu_q_lens", cu_q_lens, torch.int32, 1)
    _dev("page_table", page_table, torch.int32, 2)
    _dev("seq_lens", seq_lens, torch.int32, 1)
    T, Hq, D = q.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    st = _lib.paged_prefill_chunk_attention(
        ctypes.byref(cache.c_struct), _ptr(q), Hq, Hq // cache.num_kv_heads, _ptr(cu_q_lens),
        _ptr(page_table), page_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], T,
        int(max_q_len), float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream))
    _check("paged_prefill_chunk_attention", st)
    return out, lse


def paged_decode_attention_noalloc(cache: PagedKVCache, q, page_table, seq_lens,
                                   max_seq_len: int, softmax_scale: Optional[float] = None,
                                   out=None, lse=None, num_ctas: int = 0, want_lse: bool = True,
                                   stream=None):
    """Decode attention that allocates no device memory inside the library.

    For callers that cannot provide a workspace: the split partials live in a
    16 MiB scratch array inside ``libpagedkv.so`` that each GPU holds until
    the process exits.  Calls share that array, so calls that overlap on the
    GPU race; keep them on one stream.  ``out``/``lse`` are still the
    caller's (allocated here only if not given).  Same results as
    ``paged_decode_attention``.
    """
    _dev("q", q, torch.bfloat16, 3)
    _dev("page_table", page_table, torch.int32, 2)
    _dev("seq_lens", seq_lens, torch.int32, 1)
    B, Hq, D = q.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    st = _lib.paged_decode_attention_noalloc(
        ctypes.byref(cache.c_struct), _ptr(q), Hq, Hq // cache.num_kv_heads, _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, int(max_seq_len), float(softmax_scale),
        _ptr(out), _ptr(lse), int(num_ctas), _stream(stream))
    _check("paged_decode_attention_noalloc", st)
    return out, lse


def paged_attention_combine(parts, lse_parts, out=None, lse=None, stream=None):
    """Merge attention over disjoint key ranges.

    ``parts`` bf16 ``[R, B, Hq, D]`` (normalised outputs of each part),
    ``lse_parts`` fp32 ``[R, B, Hq]``.  Returns ``(out [B, Hq, D], lse [B, Hq])``.
    """
    _dev("parts", parts, torch.bfloat16, 4)
    _dev("lse_parts", lse_parts, torch.float32, 3)
    R, B, Hq, D = parts.shape
    if tuple(lse_parts.shape) != (R, B, Hq):
        raise ValueError("lse_parts must be [R, B, Hq]")
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=parts.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=parts.device)
    _check("paged_attention_combine",
           _lib.paged_attention_combine(_ptr(parts), _ptr(lse_parts), R, B * Hq, D, _ptr(out),
                                        _ptr(lse), _stream(stream)))
    return out, lse


def pkv_check_bounded_wait(error_flags, limit_ns: int = 0, waited_ns=None, stream=None) -> None:
    """Run the kernels' bounded mbarrier wait on a barrier nothing arrives on.

    ``error_flags`` int32 device scalar receives ``PKV_FLAG_TIMEOUT`` when the
    wait gives up after ``limit_ns`` (0: the kernels' own limit);
    ``waited_ns`` (optional int64 device scalar) receives the time waited.
    """
    _dev("error_flags", error_flags, torch.int32)
    if waited_ns is not None:
        _dev("waited_ns", waited_ns, torch.int64)
    _check("pkv_check_bounded_wait",
           _lib.pkv_check_bounded_wait(_ptr(error_flags), int(limit_ns), _ptr(waited_ns),
                                       _stream(stream)))


# ----------------------------------------------------- host runtime (paged_kv_runtime.h)
def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class PageAllocator:
    """The library's host page allocator (``pkv_allocator``) for one pool.

    Free pages form a stack (``page_order[0]`` on top); growing a slot pops
    pages in logical order, releasing pushes them back so the slot's first page
    ends on top; growth is all-or-nothing.  ``table`` is a live numpy view of
    the allocator's ``[max_seqs][max_pages_per_seq]`` page table.
    """

    def __init__(self, num_pages: int, page_size: int, max_seqs: int, max_pages_per_seq: int,
                 page_order: Optional[np.ndarray] = None):
        order = None
        if page_order is not None:
            order = np.ascontiguousarray(page_order, dtype=np.int32)
            if order.shape != (num_pages,):
                raise ValueError("page_order must have num_pages entries")
        h = ctypes.c_void_p()
        _check("pkv_allocator_create",
               _lib.pkv_allocator_create(num_pages, page_size, max_seqs, max_pages_per_seq,
                                         None if order is None else _i32p(order),
                                         ctypes.byref(h)))
        self._h = h
        self._destroy = _lib.pkv_allocator_destroy  # usable during interpreter shutdown
        self.num_pages, self.page_size = num_pages, page_size
        self.max_seqs, self.max_pages_per_seq = max_seqs, max_pages_per_seq

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def grow(self, slot: int, new_len: int) -> int:
        """Grow ``slot`` to ``new_len`` tokens; returns the status (0 or PKV_ERR_NO_PAGES)."""
        st = _lib.pkv_allocator_grow(self._h, slot, new_len)
        if st not in (0, PKV_ERR_NO_PAGES):
            _check("pkv_allocator_grow", st)
        return st

    def release(self, slot: int):
        _check("pkv_allocator_release", _lib.pkv_allocator_release(self._h, slot))

    def seq_len(self, slot: int) -> int:
        v = ctypes.c_int32()
        _check("pkv_allocator_seq_len", _lib.pkv_allocator_seq_len(self._h, slot, ctypes.byref(v)))
        return v.value

    @property
    def table(self) -> np.ndarray:
        p = _lib.pkv_allocator_table(self._h)
        return np.ctypeslib.as_array(p, shape=(self.max_seqs, self.max_pages_per_seq))

    def stats(self) -> AllocStats:
        s = AllocStats()
        _check("pkv_allocator_stats", _lib.pkv_allocator_stats(self._h, ctypes.byref(s)))
        return s

    def free_pages(self) -> np.ndarray:
        """The free stack, top first."""
        n = ctypes.c_int32()
        out = np.empty(self.num_pages, dtype=np.int32)
        _check("pkv_allocator_free_pages",
               _lib.pkv_allocator_free_pages(self._h, _i32p(out), self.num_pages, ctypes.byref(n)))
        return out[: n.value].copy()

    def step_plan(self, slots, new_tokens):
        """Plan one in-flight step (see ``pkv_step_plan``).

        Returns ``(status, plan)``; ``plan`` is a dict of host int32 arrays
        ``seq_lens_before [n]``, ``cu_new [n+1]``, ``seq_lens_after [n]`` and
        ``page_table [n][max_pages_per_seq]``, or None on PKV_ERR_NO_PAGES.
        """
        slots = np.ascontiguousarray(slots, dtype=np.int32)
        new = np.ascontiguousarray(new_tokens, dtype=np.int32)
        n = len(slots)
        if new.shape != (n,):
            raise ValueError("slots and new_tokens must have the same length")
        before = np.empty(n, np.int32)
        cu = np.empty(n + 1, np.int32)
        after = np.empty(n, np.int32)
        table = np.empty((n, self.max_pages_per_seq), np.int32)
        st = _lib.pkv_step_plan(self._h, _i32p(slots), _i32p(new), n, _i32p(before), _i32p(cu),
                                _i32p(after), _i32p(table))
        if st == PKV_ERR_NO_PAGES:
            return st, None
        _check("pkv_step_plan", st)
        return 0, {"seq_lens_before": before, "cu_new": cu, "seq_lens_after": after,
                   "page_table": table}


class StepDriver:
    """One in-flight step on the library: plan pages, stage, append, attend.

    Rows of a step are ordered decode rows first (one new token each), then
    prefill chunks.  ``pkv_step_plan`` writes the step's lengths, prefix sums
    and page-table rows straight into one pinned host buffer, one
    host-to-device copy moves it, and the step runs ``paged_kv_append`` over
    all rows, ``paged_decode_attention`` over the decode rows and
    ``paged_prefill_chunk_attention`` over the chunks, on one stream.
    """

    def __init__(self, cache: PagedKVCache, allocator: PageAllocator, max_rows: int,
                 device="cuda"):
        self.cache, self.alloc = cache, allocator
        self.max_rows = int(max_rows)
        mp = allocator.max_pages_per_seq
        n = self.max_rows
        words = 4 * n + 2 + n * mp
        self._host = torch.empty(words, dtype=torch.int32, pin_memory=True)
        self._dev = torch.empty(words, dtype=torch.int32, device=device)
        self._slots = np.empty(n, np.int32)
        self._new = np.empty(n, np.int32)
        self._copied = None  # event: the staging buffer's last copy is done
        self.device = device

    def step(self, decode_slots, chunk_slots, chunk_lens, k_new, v_new, q_decode=None,
             q_chunks=None, softmax_scale=None, stream=None):
        """Run one step; returns ``(status, decode (out, lse) or None, chunks (out, lse) or None)``.

        ``k_new``/``v_new``: bf16 ``[T, Hkv, D]`` on the device, the decode
        rows' tokens first, then each chunk's tokens.  On PKV_ERR_NO_PAGES
        nothing is launched and the allocator is unchanged.
        """
        nd, nc = len(decode_slots), len(chunk_slots)
        n = nd + nc
        if n == 0 or n > self.max_rows:
            raise ValueError(f"a step needs 1..{self.max_rows} rows, got {n}")
        mp = self.alloc.max_pages_per_seq
        self._slots[:nd] = decode_slots
        self._slots[nd:n] = chunk_slots
        self._new[:nd] = 1
        self._new[nd:n] = chunk_lens
        if self._copied is not None:
            self._copied.synchronize()  # the previous step's copy still reads the buffer
        h = self._host.numpy()
        before, cu = h[0:n], h[n:2 * n + 1]
        after, table = h[2 * n + 1:3 * n + 1], h[3 * n + 1:3 * n + 1 + n * mp]
        cu_q = h[3 * n + 1 + n * mp:3 * n + 1 + n * mp + nc + 1]
        st = _lib.pkv_step_plan(self.alloc._h, _i32p(self._slots), _i32p(self._new), n,
                                _i32p(before), _i32p(cu), _i32p(after), _i32p(table))
        if st == PKV_ERR_NO_PAGES:
            return st, None, None
        _check("pkv_step_plan", st)
        cu_q[:] = cu[nd:n + 1] - cu[nd]  # the chunks' own prefix sums
        words = 3 * n + 2 + n * mp + nc
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            d = self._dev[:words]
            d.copy_(self._host[:words], non_blocking=True)
            self._copied = torch.cuda.Event()
            self._copied.record(s)
            d_before, d_cu = d[0:n], d[n:2 * n + 1]
            d_after = d[2 * n + 1:3 * n + 1]
            d_table = d[3 * n + 1:3 * n + 1 + n * mp].view(n, mp)
            d_cu_q = d[3 * n + 1 + n * mp:]
            total = int(cu[n])
            paged_kv_append(self.cache, d_table, d_before, d_cu, k_new, v_new,
                            total_new_tokens=total, stream=s)
            dec = chk = None
            if nd:
                dec = paged_decode_attention(self.cache, q_decode, d_table[:nd], d_after[:nd],
                                             int(after[:nd].max()), softmax_scale, stream=s)
            if nc:
                chk = paged_prefill_chunk_attention(self.cache, q_chunks, d_cu_q, d_table[nd:],
                                                    d_after[nd:], int(self._new[nd:n].max()),
                                                    softmax_scale, stream=s)
        return 0, dec, chk
