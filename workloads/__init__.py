"""Seeded synthetic workloads for attention over a paged KV cache.

This module only *generates inputs*: sequence lengths, the assignment of
physical pages to sequences, page tables, and bf16 Q/K/V values (plus the
caller-side FP8 scale policy, absmax/448 per page and KV head).  It computes
no part of the attention method itself, so both the CUDA path and the CPU
oracle can consume the same inputs without sharing any of the method's
arithmetic.

Structure and values follow the workloads of the paged-attention pages
(TensorRT-LLM concept page, "PagedAttention 及 KV 快取管理": fixed-size pages
of 64 or 128 tokens mapped through a per-sequence page table) and the five
benchmark shapes of this library:

1. tiny decode        4 seqs {17,64,100,130}, P=64, 16-page pool, 8/8 heads, D=64
2. Llama-3-8B decode  64 seqs U[128,4096], P=64, pool = pages+10%, 32/8, D=128
3. long-context       8 seqs U[32768,131072], P=128, exact pool, 32/8, D=128
4. 70B FP8 decode     256 seqs lognormal(median 1024, sigma 0.8) <= 8191 ctx,
                      P=64, 64/8, D=128, E4M3 K/V with per-(page, head) scale
5. in-flight mixed    32 decode U[256,4096] + 4 chunks of 512 new tokens over
                      ctx U[0,2048], P=64, 32/8, D=128
6, 7.                 config 4's batch with INT8, and with FP4 (E2M1 + E4M3
                      block scales), K/V pools

Recipe (identical for every config):
* ``numpy.random.default_rng(seed)`` draws the context lengths first, then one
  permutation of the physical page ids; sequence ``b`` takes its logical pages
  in order from that permutation.
* Values: ``torch.Generator('cpu')`` seeded per (seed, stream, sequence) draws
  ``randn`` in fp32, rounded to bf16 (round-to-nearest-even).  Each sequence's
  K/V can therefore be regenerated on its own, which lets a checker rebuild a
  sample of sequences without materialising the whole pool.
* Context lengths are the tokens *before* this step's append; attention sees
  ``ctx + new`` tokens.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable, Optional, Sequence

import numpy as np
import torch

# Sentinels written into every pool byte that no sequence owns (bf16 quiet NaN
# and the E4M3 NaN code).  Any stray read of them turns an output into NaN.
BF16_NAN_BITS = 0x7FC0
E4M3_NAN_CODE = 0x7F
E4M3_MAX = 448.0
# INT8 pools: -128 is never stored (codes are clamped to +-127), so it marks
# bytes no sequence owns.
INT8_UNOWNED = 0x80
INT8_MAX = 127.0
# FP4 pools (E2M1 codes + E4M3 block scales): the per-(page, kv head) scale
# divides by 448 * 6 so that block scales stay within E4M3's range; unowned
# bytes hold 0x7F, whose block scale reads as NaN.
NVFP4_SCALE_DIV = E4M3_MAX * 6.0


def sentinel_byte(kv_dtype: str) -> int:
    """Fill byte of unowned pool bytes of a one-byte or FP4 pool."""
    return {"e4m3": E4M3_NAN_CODE, "int8": INT8_UNOWNED, "nvfp4": E4M3_NAN_CODE}[kv_dtype]


def code_max(kv_dtype: str) -> float:
    """Largest stored magnitude of a format relative to its scale (the divisor)."""
    return {"e4m3": E4M3_MAX, "int8": INT8_MAX, "nvfp4": NVFP4_SCALE_DIV}[kv_dtype]

_STREAM_KV = 1
_STREAM_QDEC = 2
_STREAM_QCHUNK = 3


def _torch_gen(seed: int, stream: int, index: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int((int(seed) * 1_000_003 + int(stream) * 65_537 + int(index)) % (2**63 - 1)))
    return g


def _randn_bf16(shape: Sequence[int], gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


@dataclasses.dataclass
class Workload:
    """One step of an in-flight batch over a paged KV pool.

    Sequences ``decode_rows`` append one token and run decode attention;
    sequences ``chunk_rows`` append a prefill chunk and run causal chunk
    attention.  All sequences share one physical pool.
    """

    name: str
    seed: int
    page_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_dtype: str  # "bf16", "e4m3", "int8" or "nvfp4"
    ctx_lens: np.ndarray  # int32 [B], tokens already cached
    new_lens: np.ndarray  # int32 [B], tokens appended this step
    num_pages: int
    page_table: np.ndarray  # int32 [B, max_pages_per_seq], -1 past the last page
    decode_rows: np.ndarray  # int64 indices into [0, B)
    chunk_rows: np.ndarray  # int64 indices into [0, B)
    softmax_scale: float
    config_number: Optional[int] = None  # set by config(n) for the numbered workloads

    # ------------------------------------------------------------ structure
    @property
    def batch(self) -> int:
        return int(self.ctx_lens.shape[0])

    @property
    def lens_after(self) -> np.ndarray:
        return (self.ctx_lens + self.new_lens).astype(np.int32)

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def gqa_group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return 2 if self.kv_dtype == "bf16" else 1

    def cu_new(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.new_lens)]).astype(np.int32)

    def pool_shape(self):
        return (self.num_pages, self.num_kv_heads, self.page_size, self.head_dim)

    def pool_bytes(self) -> int:
        if self.kv_dtype == "nvfp4":  # codes (D/2 a row) then block scales (D/16 a row)
            rows = self.num_pages * self.num_kv_heads * self.page_size
            return rows * (self.head_dim // 2 + self.head_dim // 16)
        return int(np.prod(self.pool_shape())) * self.elem_bytes

    def pages_of(self, b: int) -> np.ndarray:
        n = -(-int(self.lens_after[b]) // self.page_size)
        return self.page_table[b, :n]

    # --------------------------------------------------------------- values
    def kv_seq(self, b: int):
        """(K, V) bf16 ``[ctx+new, Hkv, D]`` of sequence ``b`` (all its tokens)."""
        n = int(self.lens_after[b])
        g = _torch_gen(self.seed, _STREAM_KV, b)
        k = _randn_bf16((n, self.num_kv_heads, self.head_dim), g)
        v = _randn_bf16((n, self.num_kv_heads, self.head_dim), g)
        return k, v

    def q_decode(self) -> torch.Tensor:
        """Decode queries, bf16 ``[len(decode_rows), Hq, D]``."""
        g = _torch_gen(self.seed, _STREAM_QDEC, 0)
        return _randn_bf16((len(self.decode_rows), self.num_q_heads, self.head_dim), g)

    def q_chunks(self) -> torch.Tensor:
        """Prefill-chunk queries packed over chunks, bf16 ``[sum new, Hq, D]``."""
        g = _torch_gen(self.seed, _STREAM_QCHUNK, 0)
        t = int(self.new_lens[self.chunk_rows].sum()) if len(self.chunk_rows) else 0
        return _randn_bf16((t, self.num_q_heads, self.head_dim), g)

    def cu_q_chunks(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.new_lens[self.chunk_rows])]).astype(np.int32)

    def new_kv(self, rows: Optional[Iterable[int]] = None):
        """Tokens appended this step, concatenated over ``rows`` (default all)."""
        rows = range(self.batch) if rows is None else rows
        ks, vs = [], []
        for b in rows:
            k, v = self.kv_seq(b)
            c = int(self.ctx_lens[b])
            ks.append(k[c:])
            vs.append(v[c:])
        if not ks:
            z = torch.empty((0, self.num_kv_heads, self.head_dim), dtype=torch.bfloat16)
            return z, z.clone()
        return torch.cat(ks), torch.cat(vs)

    # ------------------------------------------------------ FP8 scale policy
    def kv_scales_for(self, b: int, k: torch.Tensor = None, v: torch.Tensor = None):
        """Per-(page, kv head) scales of sequence ``b``: absmax/448 (E4M3),
        absmax/127 (INT8) or absmax/(448*6) (FP4) in fp32.

        The absmax runs over every element the page will hold after this
        step's append, so no stored value saturates.  Returns
        ``(page_ids, k_scale[n_pages, Hkv], v_scale[n_pages, Hkv])``.
        """
        if k is None:
            k, v = self.kv_seq(b)
        pages = self.pages_of(b)
        n = k.shape[0]
        P = self.page_size
        ks = np.empty((len(pages), self.num_kv_heads), np.float32)
        vs = np.empty((len(pages), self.num_kv_heads), np.float32)
        for j in range(len(pages)):
            lo, hi = j * P, min((j + 1) * P, n)
            ka = k[lo:hi].float().abs().amax(dim=(0, 2)).numpy().astype(np.float32)
            va = v[lo:hi].float().abs().amax(dim=(0, 2)).numpy().astype(np.float32)
            ks[j] = ka / np.float32(code_max(self.kv_dtype))
            vs[j] = va / np.float32(code_max(self.kv_dtype))
        tiny = np.float32(2.0**-126)
        return pages, np.maximum(ks, tiny), np.maximum(vs, tiny)

    def kv_scales(self):
        """Full ``[num_pages, Hkv]`` fp32 K and V scale tables (1.0 on unowned pages)."""
        ks = np.ones((self.num_pages, self.num_kv_heads), np.float32)
        vs = np.ones((self.num_pages, self.num_kv_heads), np.float32)
        for b in range(self.batch):
            pages, k_s, v_s = self.kv_scales_for(b)
            ks[pages] = k_s
            vs[pages] = v_s
        return ks, vs

    # ---------------------------------------------------------- byte counts
    def decode_kv_tokens(self) -> int:
        return int(self.lens_after[self.decode_rows].sum())

    def describe(self) -> dict:
        la = self.lens_after
        return {
            "workload": self.name,
            "seed": self.seed,
            "batch": self.batch,
            "decode_seqs": int(len(self.decode_rows)),
            "prefill_chunks": int(len(self.chunk_rows)),
            "page_size": self.page_size,
            "num_q_heads": self.num_q_heads,
            "num_kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim,
            "kv_dtype": self.kv_dtype,
            "num_pages": self.num_pages,
            "tokens_after_append": int(la.sum()),
            "min_len": int(la.min()) if len(la) else 0,
            "max_len": int(la.max()) if len(la) else 0,
        }


# ------------------------------------------------------------------ builders
def build(
    name: str,
    seed: int,
    ctx_lens: Sequence[int],
    new_lens: Sequence[int],
    *,
    page_size: int,
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    kv_dtype: str = "bf16",
    pool_pages: Optional[int] = None,
    pool_slack: float = 0.0,
    chunk_rows: Sequence[int] = (),
    softmax_scale: Optional[float] = None,
    rng: Optional[np.random.Generator] = None,
    max_pages_per_seq: Optional[int] = None,
) -> Workload:
    """Assign permuted physical pages to sequences and build the page table."""
    rng = np.random.default_rng(seed) if rng is None else rng
    ctx = np.asarray(ctx_lens, dtype=np.int32)
    new = np.asarray(new_lens, dtype=np.int32)
    after = ctx.astype(np.int64) + new
    need = -(-after // page_size)
    total = int(need.sum())
    if pool_pages is None:
        pool_pages = int(math.ceil(total * (1.0 + pool_slack))) if pool_slack else total
    if pool_pages < total:
        raise ValueError(f"pool of {pool_pages} pages cannot hold {total}")
    perm = rng.permutation(pool_pages).astype(np.int32)
    maxp = int(need.max()) if len(need) else 1
    if max_pages_per_seq is not None:
        maxp = max(maxp, max_pages_per_seq)
    maxp = max(maxp, 1)
    table = np.full((len(ctx), maxp), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off : off + n]
        off += int(n)
    chunk = np.asarray(sorted(chunk_rows), dtype=np.int64)
    dec = np.asarray([b for b in range(len(ctx)) if b not in set(chunk.tolist())], dtype=np.int64)
    scale = 1.0 / math.sqrt(head_dim) if softmax_scale is None else float(softmax_scale)
    return Workload(
        name=name,
        seed=seed,
        page_size=page_size,
        num_q_heads=num_q_heads,
        num_kv_heads=num_kv_heads,
        head_dim=head_dim,
        kv_dtype=kv_dtype,
        ctx_lens=ctx,
        new_lens=new,
        num_pages=pool_pages,
        page_table=table,
        decode_rows=dec,
        chunk_rows=chunk,
        softmax_scale=scale,
    )


def tiny_decode(seed: int = 0) -> Workload:
    """4 seqs of context {17,64,100,130}, P=64, 16-page pool, 8/8 heads, D=64."""
    return build("tiny_decode_b4_p64_h8_d64", seed, [17, 64, 100, 130], [1] * 4,
                 page_size=64, num_q_heads=8, num_kv_heads=8, head_dim=64,
                 pool_pages=16, softmax_scale=1.0 / 8.0)


def llama8b_decode(seed: int = 1) -> Workload:
    """64 seqs, context U[128,4096], P=64, pool = pages + 10%, 32/8 heads, D=128."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(128, 4096 + 1, size=64)
    return build("llama3_8b_decode_b64_p64_gqa4_d128", seed, ctx, [1] * 64,
                 page_size=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 pool_slack=0.10, rng=rng)


def long_context_decode(seed: int = 2) -> Workload:
    """8 seqs, context U[32768,131072], P=128, exact pool, 32/8 heads, D=128."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(32768, 131072 + 1, size=8)
    return build("long_ctx_decode_b8_p128_gqa4_d128", seed, ctx, [1] * 8,
                 page_size=128, num_q_heads=32, num_kv_heads=8, head_dim=128, rng=rng)


def llama70b_fp8_decode(seed: int = 3) -> Workload:
    """256 seqs, context lognormal(median 1024, sigma 0.8) capped so L<=8192, E4M3 K/V."""
    rng = np.random.default_rng(seed)
    ctx = np.clip(np.rint(np.exp(rng.normal(math.log(1024.0), 0.8, size=256))), 1, 8191)
    return build("llama3_70b_fp8_decode_b256_p64_gqa8_d128", seed, ctx.astype(np.int64), [1] * 256,
                 page_size=64, num_q_heads=64, num_kv_heads=8, head_dim=128,
                 kv_dtype="e4m3", rng=rng)


def llama70b_int8_decode(seed: int = 3) -> Workload:
    """The 70B-shaped decode batch of ``llama70b_fp8_decode`` with INT8 K/V pools."""
    rng = np.random.default_rng(seed)
    ctx = np.clip(np.rint(np.exp(rng.normal(math.log(1024.0), 0.8, size=256))), 1, 8191)
    return build("llama3_70b_int8_decode_b256_p64_gqa8_d128", seed, ctx.astype(np.int64),
                 [1] * 256, page_size=64, num_q_heads=64, num_kv_heads=8, head_dim=128,
                 kv_dtype="int8", rng=rng)


def llama70b_nvfp4_decode(seed: int = 3) -> Workload:
    """The 70B-shaped decode batch of ``llama70b_fp8_decode`` with FP4 K/V pools
    (E2M1 codes, E4M3 block scales per 16 values, per-(page, head) scale)."""
    rng = np.random.default_rng(seed)
    ctx = np.clip(np.rint(np.exp(rng.normal(math.log(1024.0), 0.8, size=256))), 1, 8191)
    return build("llama3_70b_nvfp4_decode_b256_p64_gqa8_d128", seed, ctx.astype(np.int64),
                 [1] * 256, page_size=64, num_q_heads=64, num_kv_heads=8, head_dim=128,
                 kv_dtype="nvfp4", rng=rng)


def mixed_inflight(seed: int = 4) -> Workload:
    """32 decode seqs U[256,4096] + 4 prefill chunks of 512 over context U[0,2048]."""
    rng = np.random.default_rng(seed)
    dec = rng.integers(256, 4096 + 1, size=32)
    chk = rng.integers(0, 2048 + 1, size=4)
    ctx = np.concatenate([dec, chk])
    new = np.array([1] * 32 + [512] * 4)
    return build("mixed_inflight_32dec_4x512chunk_p64_gqa4_d128", seed, ctx, new,
                 page_size=64, num_q_heads=32, num_kv_heads=8, head_dim=128,
                 chunk_rows=range(32, 36), rng=rng)


CONFIGS = {
    1: tiny_decode,
    2: llama8b_decode,
    3: long_context_decode,
    4: llama70b_fp8_decode,
    5: mixed_inflight,
    6: llama70b_int8_decode,
    7: llama70b_nvfp4_decode,
}


def config(n: int, seed: Optional[int] = None) -> Workload:
    fn = CONFIGS[n]
    w = fn() if seed is None else fn(seed)
    w.config_number = n
    return w


def empty_pool(w: Workload) -> np.ndarray:
    """Host pool image (uint8 view) filled with the NaN sentinel of its dtype."""
    if w.kv_dtype != "bf16":
        return np.full(w.pool_bytes(), sentinel_byte(w.kv_dtype), dtype=np.uint8)
    return np.full(w.pool_bytes() // 2, BF16_NAN_BITS, dtype=np.uint16).view(np.uint8)
