"""Sharding the paged attention over GPUs (one process per GPU).

Two ways the path splits, from the shapes of the work (concept page,
"PagedAttention 及 KV 快取管理": a sequence's K/V is a list of pages, each
page holding every kv head of its tokens; column-parallel attention keeps
whole heads on one device):

* **by kv head** (``head_shard``): rank r keeps kv heads
  ``[r*Hkv/N, (r+1)*Hkv/N)`` of every page and the q heads that read them.
  Each rank runs the ordinary calls on its own pools; the outputs are
  disjoint head slices and nothing is exchanged.
* **by page range** (``page_split`` + ``decode_sequence_parallel``): a long
  sequence's pages are cut into N contiguous ranges.  Each rank attends over
  its range (its slice of the page-table row, length = its tokens) and the
  partial results -- normalised output and log-sum-exp -- are all-gathered
  and merged by ``paged_attention_combine``.  This is the one exchange the
  path has: B * Hq * (D * 2 + 4) bytes per rank.

The host arithmetic here is plain integer work; the attention and the merge
run in the library's kernels.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np
import torch

from . import paged_attention_combine, paged_decode_attention


def head_shard(num_q_heads: int, num_kv_heads: int, world: int, rank: int) -> Tuple[int, int, int, int]:
    """(q_lo, q_hi, kv_lo, kv_hi) of rank ``rank``: contiguous kv-head blocks
    and the q heads that read them (q head h reads kv head h // G)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if num_kv_heads % world:
        raise ValueError(f"{num_kv_heads} kv heads do not split over {world} ranks")
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    per = num_kv_heads // world
    G = num_q_heads // num_kv_heads
    kv_lo, kv_hi = rank * per, (rank + 1) * per
    return kv_lo * G, kv_hi * G, kv_lo, kv_hi


def page_split(seq_lens, page_size: int, world: int, rank: int):
    """Rank ``rank``'s share of every sequence: a contiguous page range.

    The ``ceil(L / P)`` pages of a sequence are cut into ``world`` ranges of
    near-equal page counts (the first ``pages % world`` ranges get one more).
    Returns ``(page_begin [B], page_end [B], local_len [B])`` as int32 arrays;
    ``local_len`` counts the tokens of the range (the last range of a
    sequence ends at L) and is 0 for an empty range.
    """
    lens = np.asarray(seq_lens, dtype=np.int64)
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    pages = -(-lens // page_size)
    base, extra = pages // world, pages % world
    begin = rank * base + np.minimum(rank, extra)
    end = begin + base + (rank < extra)
    tok_begin = np.minimum(begin * page_size, lens)
    tok_end = np.minimum(end * page_size, lens)
    return (begin.astype(np.int32), end.astype(np.int32),
            (tok_end - tok_begin).astype(np.int32))


def local_table(page_table: torch.Tensor, page_begin, page_end) -> torch.Tensor:
    """Rows of ``page_table`` shifted to start at each sequence's first page of
    the range (entries past the range are -1), on the table's device."""
    rows = page_table.shape[0]
    width = max(1, int(np.max(np.asarray(page_end) - np.asarray(page_begin), initial=0)))
    host = page_table.cpu().numpy()
    out = np.full((rows, width), -1, dtype=np.int32)
    for b in range(rows):
        n = int(page_end[b]) - int(page_begin[b])
        out[b, :n] = host[b, int(page_begin[b]):int(page_end[b])]
    return torch.from_numpy(out).to(page_table.device)


def decode_sequence_parallel(cache, q, page_table_local, local_lens, max_local_len: int,
                             softmax_scale, group=None, out=None, lse=None):
    """Decode with each sequence's pages split over the ranks of ``group``.

    Every rank passes its own cache (its pages), its slice of the page table
    (``local_table``) and its token counts (``page_split``).  The partial
    outputs and lse are all-gathered over ``torch.distributed`` (NCCL on GPUs)
    and merged by ``paged_attention_combine``; every rank returns the full
    result.
    """
    import torch.distributed as dist

    part, part_lse = paged_decode_attention(cache, q, page_table_local, local_lens,
                                            max_local_len, softmax_scale)
    world = dist.get_world_size(group)
    parts = torch.empty((world,) + tuple(part.shape), dtype=part.dtype, device=part.device)
    lses = torch.empty((world,) + tuple(part_lse.shape), dtype=part_lse.dtype,
                       device=part.device)
    dist.all_gather_into_tensor(parts, part.contiguous(), group=group)
    dist.all_gather_into_tensor(lses, part_lse.contiguous(), group=group)
    return paged_attention_combine(parts, lses, out=out, lse=lse)
