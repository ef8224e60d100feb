"""Multi-GPU shardings of the path, each rank run in turn on one GPU.

The ranks of both shardings are independent until the exchange (no kernel
waits on another rank), so running them one after another on one device
gives exactly what N devices would compute; the exchange itself is an
all-gather, here a stack.

* by kv head: every rank owns its heads' slice of every page in pools of its
  own, filled by the library's append; its decode output is the matching
  head slice of the oracle's full decode;
* by page range: every rank attends over its pages of each sequence through
  its slice of the page table; ``paged_attention_combine`` merges the
  partials and must match the oracle's full decode;
* the combine kernel: one part returns that part bit for bit, empty parts
  weigh nothing, a row with no key at all is 0 with lse -inf.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu


def _oracle_decode(w):
    c = oracle.cache_for(w)
    return c.decode(oracle.bf16_bits(w.q_decode()), w.page_table, w.lens_after, w.softmax_scale)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_head_sharded_decode(world, dtype):
    import paged_kv_cache_476_b200 as pkv
    from paged_kv_cache_476_b200.parallel import head_shard

    w = workloads.build("hs", 51, [0, 40, 700, 2047, 3000], [1] * 5, page_size=64,
                        num_q_heads=32, num_kv_heads=8, head_dim=128, kv_dtype=dtype,
                        pool_slack=0.2)
    full = GpuState(w)  # the whole pool, filled through the library's append
    full.append_step()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    q = w.q_decode().cuda()
    table = full.table
    lens = torch.from_numpy(w.lens_after).cuda()
    for r in range(world):
        q_lo, q_hi, kv_lo, kv_hi = head_shard(32, 8, world, r)
        # this rank's pools hold its kv heads of every page
        kp = full.k_pool[:, kv_lo:kv_hi].contiguous()
        vp = full.v_pool[:, kv_lo:kv_hi].contiguous()
        ks = vs = None
        if dtype != "bf16":
            ks = full.k_scale[:, kv_lo:kv_hi].contiguous()
            vs = full.v_scale[:, kv_lo:kv_hi].contiguous()
        cache = pkv.PagedKVCache(kp, vp, dtype, ks, vs, full.flags)
        out, lse = pkv.paged_decode_attention(cache, q[:, q_lo:q_hi].contiguous(), table, lens,
                                              int(w.lens_after.max()), w.softmax_scale)
        torch.cuda.synchronize()
        compare(out, lse, ref[:, q_lo:q_hi], ref_lse[:, q_lo:q_hi])
    assert int(full.flags.item()) == 0


@pytest.mark.parametrize("world", [2, 3, 8])
def test_page_split_decode_with_combine(world):
    import paged_kv_cache_476_b200 as pkv
    from paged_kv_cache_476_b200.parallel import local_table, page_split

    w = workloads.build("sp", 52, [0, 63, 64, 1000, 9000, 33000], [1] * 6, page_size=128,
                        num_q_heads=32, num_kv_heads=8, head_dim=128, pool_slack=0.1)
    st = GpuState(w)
    st.append_step()
    q = w.q_decode().cuda()
    parts, lses = [], []
    for r in range(world):
        begin, end, local = page_split(w.lens_after, w.page_size, world, r)
        table = local_table(st.table, begin, end)
        out, lse = pkv.paged_decode_attention(st.cache, q, table,
                                              torch.from_numpy(local).cuda(),
                                              max(1, int(local.max())), w.softmax_scale)
        parts.append(out)
        lses.append(lse)
    out, lse = pkv.paged_attention_combine(torch.stack(parts), torch.stack(lses))
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


def test_combine_edge_cases():
    import paged_kv_cache_476_b200 as pkv

    g = torch.Generator().manual_seed(5)
    part = torch.randn(1, 3, 4, 128, generator=g).to(torch.bfloat16).cuda()
    lse = torch.randn(1, 3, 4, generator=g).cuda()
    out, l2 = pkv.paged_attention_combine(part, lse)
    torch.cuda.synchronize()
    assert torch.equal(out, part[0]) and torch.equal(l2, lse[0])  # one part: itself
    # an empty part (lse -inf, garbage output) weighs nothing
    junk = torch.full_like(part, 1e4)
    both = torch.cat([part, junk])
    both_lse = torch.cat([lse, torch.full_like(lse, float("-inf"))])
    out, l2 = pkv.paged_attention_combine(both, both_lse)
    torch.cuda.synchronize()
    assert torch.equal(out, part[0]) and torch.equal(l2, lse[0])
    # a row no part saw: 0 with lse -inf
    none_lse = torch.full((2, 3, 4), float("-inf")).cuda()
    out, l2 = pkv.paged_attention_combine(both[:, :, :, :64].contiguous(), none_lse)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(l2))
    # two equal parts: the same output, lse + ln 2
    out, l2 = pkv.paged_attention_combine(torch.cat([part, part]), torch.cat([lse, lse]))
    torch.cuda.synchronize()
    assert torch.equal(out, part[0])
    assert torch.allclose(l2, lse[0] + np.log(2.0), atol=1e-6)
