"""Pure-Python brute force of paged attention, for tiny inputs only.

An independent restatement of the definition used to pin the C oracle: it
walks the page table token by token with plain Python integers, decodes bf16
bits with ``struct``, E4M3 codes (and FP4 block scales) through torch's
``float8_e4m3fn`` (a library routine), E2M1 codes through the format's
value table, and sums with ``math.fsum``.  It shares nothing with
``oracle/oracle.c``.
"""
from __future__ import annotations

import math
import struct

import numpy as np
import torch


def bf16_to_float(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


_E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(
    torch.float64).tolist()


def e4m3_to_float(code: int) -> float:
    return _E4M3[int(code)]


# E2M1 magnitudes in code order (sign in bit 3), from the format definition
_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def element(cache, pool, scales, page, g, slot, d) -> float:
    """Value of one stored K or V element, read from the raw byte pool."""
    H, P, D = cache.num_kv_heads, cache.page_size, cache.head_dim
    row = (page * H + g) * P + slot
    if cache.kv_dtype == "nvfp4":  # code region, then block-scale region
        byte = int(pool[row * (D // 2) + d // 2])
        code = (byte >> 4) if d % 2 else (byte & 0xF)
        mag = _E2M1[code & 7]
        sb = int(pool[cache.num_pages * H * P * (D // 2) + row * (D // 16) + d // 16])
        return (-mag if code & 8 else mag) * e4m3_to_float(sb) * float(scales[page, g])
    idx = row * D + d
    if cache.kv_dtype == "e4m3":
        return e4m3_to_float(pool[idx]) * float(scales[page, g])
    if cache.kv_dtype == "int8":  # two's-complement byte times the scale
        code = int(pool[idx])
        return float(code - 256 if code > 127 else code) * float(scales[page, g])
    lo, hi = int(pool[2 * idx]), int(pool[2 * idx + 1])
    return bf16_to_float(lo | (hi << 8))


def kv_rows(cache, table_row, n, g):
    K, V = [], []
    for t in range(n):
        page = int(table_row[t // cache.page_size])
        slot = t % cache.page_size
        K.append([element(cache, cache.k_pool, cache.k_scale, page, g, slot, d)
                  for d in range(cache.head_dim)])
        V.append([element(cache, cache.v_pool, cache.v_scale, page, g, slot, d)
                  for d in range(cache.head_dim)])
    return K, V


def attend(q, K, V, scale):
    """Textbook softmax(scale * q.K) V with fsum; returns (o, lse)."""
    n = len(K)
    if n == 0:
        return [0.0] * len(q), -math.inf
    s = [scale * math.fsum(qi * ki for qi, ki in zip(q, krow)) for krow in K]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    den = math.fsum(e)
    o = [math.fsum(e[t] * V[t][d] for t in range(n)) / den for d in range(len(q))]
    return o, m + math.log(den)


def decode(cache, q_bits, page_table, seq_lens, scale):
    B, Hq, D = q_bits.shape
    G = Hq // cache.num_kv_heads
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            K, V = kv_rows(cache, page_table[b], int(seq_lens[b]), h // G)
            q = [bf16_to_float(x) for x in q_bits[b, h]]
            o, l = attend(q, K, V, scale)
            out[b, h] = o
            lse[b, h] = l
    return out, lse


def prefill_chunk(cache, q_bits, cu_q, page_table, seq_lens, scale):
    T, Hq, D = q_bits.shape
    G = Hq // cache.num_kv_heads
    out = np.zeros((T, Hq, D))
    lse = np.zeros((T, Hq))
    for c in range(len(seq_lens)):
        n = int(cu_q[c + 1] - cu_q[c])
        L = int(seq_lens[c])
        for i in range(n):
            row = int(cu_q[c]) + i
            p = L - n + i
            for h in range(Hq):
                K, V = kv_rows(cache, page_table[c], p + 1, h // G)
                q = [bf16_to_float(x) for x in q_bits[row, h]]
                o, l = attend(q, K, V, scale)
                out[row, h] = o
                lse[row, h] = l
    return out, lse
