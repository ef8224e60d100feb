"""Host logic of the multi-GPU shardings, on CPU (``gloo``, world size 2).

* ``head_shard`` covers every kv head exactly once and keeps each q head with
  the kv head it reads.
* ``page_split`` cuts each sequence's pages into contiguous ranges that
  partition them, with token counts that add up to the length.
* Two gloo ranks run the sequence-parallel protocol end to end with the
  oracle standing in for the per-rank attention: each attends over its page
  range through its slice of the page table, the partial outputs and lse are
  all-gathered in rank order, and merging them (the split-KV formula, the
  oracle's ``merge``) reproduces the unsplit oracle decode to 1e-12.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads


@pytest.fixture(scope="module")
def par():
    import __graft_entry__

    __graft_entry__._builder().build()
    from paged_kv_cache_476_b200 import parallel

    return parallel


def test_head_shard_partitions_heads(par):
    for Hq, Hkv, N in [(32, 8, 2), (32, 8, 4), (64, 8, 8), (8, 8, 2)]:
        G = Hq // Hkv
        seen_q, seen_kv = [], []
        for r in range(N):
            q_lo, q_hi, kv_lo, kv_hi = par.head_shard(Hq, Hkv, N, r)
            seen_q += list(range(q_lo, q_hi))
            seen_kv += list(range(kv_lo, kv_hi))
            assert all(kv_lo <= h // G < kv_hi for h in range(q_lo, q_hi))
        assert seen_q == list(range(Hq)) and seen_kv == list(range(Hkv))
    with pytest.raises(ValueError):
        par.head_shard(32, 8, 3, 0)


def test_page_split_partitions_pages(par):
    rng = np.random.default_rng(3)
    lens = np.concatenate([[0, 1, 63, 64, 65], rng.integers(1, 140000, size=40)])
    for P in (64, 128):
        for N in (1, 2, 3, 8):
            ranges = [par.page_split(lens, P, N, r) for r in range(N)]
            pages = -(-lens // P)
            for b in range(len(lens)):
                begins = [int(rg[0][b]) for rg in ranges]
                ends = [int(rg[1][b]) for rg in ranges]
                assert begins[0] == 0 and ends[-1] == pages[b]
                assert all(ends[r] == begins[r + 1] for r in range(N - 1))
                sizes = [e - s for s, e in zip(begins, ends)]
                assert max(sizes) - min(sizes) <= 1
                assert sum(int(rg[2][b]) for rg in ranges) == lens[b]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, result_path):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from paged_kv_cache_476_b200 import parallel

        w = workloads.build("sp", 17, [0, 5, 64, 700, 1500, 130], [1] * 6, page_size=64,
                            num_q_heads=8, num_kv_heads=2, head_dim=32, pool_slack=0.2)
        c = oracle.cache_for(w)
        q = oracle.bf16_bits(w.q_decode())
        begin, end, local = parallel.page_split(w.lens_after, w.page_size, world, rank)
        table = parallel.local_table(torch.from_numpy(w.page_table), begin, end).numpy()
        out, lse = c.decode(q, table, local, w.softmax_scale)  # this rank's pages only
        parts = [torch.empty(out.shape, dtype=torch.float64) for _ in range(world)]
        lses = [torch.empty(lse.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(out))
        dist.all_gather(lses, torch.from_numpy(lse))
        B, Hq, D = out.shape
        acc = np.stack([p.numpy() for p in parts]).reshape(world, B * Hq, D)
        m = np.stack([x.numpy() for x in lses]).reshape(world, B * Hq)
        got, got_lse = oracle.merge(acc, m, np.ones_like(m))  # normalised parts: l = 1
        ref, ref_lse = c.decode(q, w.page_table, w.lens_after, w.softmax_scale)
        err = max(np.abs(got - ref.reshape(B * Hq, D)).max(),
                  np.abs(got_lse - ref_lse.reshape(-1)).max())
        if rank == 0:
            with open(result_path, "w") as f:
                f.write(repr(float(err)))
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_protocol_on_two_gloo_ranks(par, tmp_path):
    result = str(tmp_path / "err.txt")
    mp.start_processes(_rank_main, args=(2, _free_port(), result), nprocs=2, join=True,
                       start_method="spawn")
    assert float(open(result).read()) < 1e-12
