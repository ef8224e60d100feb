"""Parity of the tcgen05 prefill-chunk kernel with the oracle (needs a GPU).

Causal chunk attention (query i of a chunk with n queries over L tokens sees
keys 0..L-n+i): bf16 output within max-abs 1e-2 and mean-abs 1e-3 of the
fp64 oracle, lse within 2e-3.  Cases cover bf16, E4M3 and INT8 pools (the
oracle attends over its own bit-identical pool of codes), GQA groups 1..8, head_dim
64/128, page sizes 64/128, chunks without context, chunks shorter than a Q
tile, ragged tails and the in-flight mixed-batch configuration.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu


def _oracle_prefill(w):
    c = oracle.cache_for(w)
    rows = w.chunk_rows
    return c.prefill_chunk(oracle.bf16_bits(w.q_chunks()), w.cu_q_chunks(), w.page_table[rows],
                           w.lens_after[rows], w.softmax_scale)


CASES = [
    # (kv dtype, P, D, Hkv, G, ctx lengths of the chunks, new tokens per chunk)
    ("bf16", 64, 128, 2, 4, [0, 100, 700], [512, 33, 130]),
    ("bf16", 64, 128, 1, 8, [5, 0], [17, 1]),
    ("bf16", 128, 128, 2, 1, [0, 129, 1000], [128, 200, 7]),
    ("bf16", 64, 64, 2, 2, [63, 64, 0], [65, 1, 300]),
    ("bf16", 128, 64, 1, 4, [300], [257]),
    ("bf16", 64, 128, 8, 4, [2048, 0, 777, 1500], [512, 512, 512, 512]),
    ("e4m3", 64, 128, 2, 4, [0, 100, 700], [512, 33, 130]),
    ("e4m3", 128, 128, 1, 8, [5, 0, 300], [17, 1, 129]),
    ("e4m3", 64, 64, 2, 2, [63, 64, 0], [65, 1, 300]),
    ("e4m3", 128, 64, 2, 1, [1000], [200]),
    ("int8", 64, 128, 2, 4, [0, 100, 700], [512, 33, 130]),
    ("int8", 128, 128, 1, 8, [5, 0, 300], [17, 1, 129]),
    ("int8", 64, 64, 2, 2, [63, 64, 0], [65, 1, 300]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-P{c[1]}-D{c[2]}-G{c[4]}")
def test_prefill_matches_oracle(case):
    dtype, P, D, Hkv, G, ctx, new = case
    w = workloads.build("pf", 21, ctx, new, page_size=P, num_q_heads=Hkv * G, num_kv_heads=Hkv,
                        head_dim=D, kv_dtype=dtype, pool_slack=0.3, chunk_rows=range(len(ctx)))
    st = GpuState(w)
    st.append_step()
    out, lse = st.prefill()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_prefill(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


@pytest.mark.parametrize("num_chunks", [128, 140])
def test_prefill_many_chunks(num_chunks):
    # up to 128 chunks the CTAs take items longest-first, beyond that in index
    # order; both must cover every (chunk, Q-tile pair, kv head) exactly once
    rng = np.random.default_rng(num_chunks)
    ctx = [int(x) for x in rng.choice([0, 7, 150, 600], size=num_chunks)]
    new = [int(x) for x in rng.choice([1, 5, 33, 64, 200], size=num_chunks)]
    w = workloads.build("pfmany", 26, ctx, new, page_size=64, num_q_heads=8, num_kv_heads=2,
                        head_dim=128, pool_slack=0.1, chunk_rows=range(num_chunks))
    st = GpuState(w)
    st.append_step()
    out, lse = st.prefill()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_prefill(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
def test_prefill_negative_scale(dtype):
    # the row max of s * scale is not scale * max(s) when scale < 0
    w = workloads.build("pfneg", 27, [300, 0], [200, 130], page_size=64, num_q_heads=8,
                        num_kv_heads=2, head_dim=128, kv_dtype=dtype, pool_slack=0.2,
                        chunk_rows=[0, 1], softmax_scale=-0.11)
    st = GpuState(w)
    st.append_step()
    out, lse = st.prefill()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_prefill(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


def test_prefill_row_equals_truncated_decode():
    # the last query of a chunk sees exactly what a decode step would see
    w = workloads.build("pfd", 22, [300, 50], [70, 9], page_size=64, num_q_heads=8,
                        num_kv_heads=2, head_dim=128, pool_slack=0.3, chunk_rows=[0, 1])
    st = GpuState(w)
    st.append_step()
    out, lse = st.prefill()
    q, cu, table, lens, _ = st.chunk_inputs()
    last = (cu[1:] - 1).long()
    d_out, d_lse = st.pkv.paged_decode_attention(st.cache, q[last].contiguous(), table, lens,
                                                 int(lens.max()), w.softmax_scale)
    torch.cuda.synchronize()
    assert (out[last].float() - d_out.float()).abs().max().item() <= 1.6e-2
    assert (lse[last] - d_lse).abs().max().item() <= 2e-3


def test_config_mixed_inflight_step():
    w = workloads.mixed_inflight()
    st = GpuState(w)
    st.append_step()
    out, lse = st.prefill()
    d_out, d_lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_prefill(w)
    compare(out, lse, ref, ref_lse)
    c = oracle.cache_for(w)
    rows = w.decode_rows
    dref, dref_lse = c.decode(oracle.bf16_bits(w.q_decode()), w.page_table[rows],
                              w.lens_after[rows], w.softmax_scale)
    compare(d_out, d_lse, dref, dref_lse)
    assert int(st.flags.item()) == 0


def test_prefill_is_deterministic():
    w = workloads.build("pfdet", 23, [1000, 10], [256, 100], page_size=64, num_q_heads=32,
                        num_kv_heads=8, head_dim=128, pool_slack=0.2, chunk_rows=[0, 1])
    st = GpuState(w)
    st.append_step()
    a, la = st.prefill()
    b, lb = st.prefill()
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_prefill_bad_page_is_masked_and_flagged():
    w = workloads.build("pfbad", 24, [200, 64], [40, 64], page_size=64, num_q_heads=4,
                        num_kv_heads=1, head_dim=128, pool_slack=0.5, chunk_rows=[0, 1])
    st = GpuState(w)
    st.append_step()
    q, cu, table, lens, max_q = st.chunk_inputs()
    table[0, 1] = w.num_pages + 3
    out, lse = st.pkv.paged_prefill_chunk_attention(st.cache, q, cu, table, lens, max_q,
                                                    w.softmax_scale)
    torch.cuda.synchronize()
    assert int(st.flags.item()) & 0x1
    assert torch.all(torch.isfinite(out.float()))
    ref, ref_lse = _oracle_prefill(w)
    rows = np.arange(int(cu[1].item()), int(cu[2].item()))
    compare(out, lse, ref, ref_lse, rows=rows)


def test_prefill_e4m3_bad_page_is_masked_and_flagged():
    w = workloads.build("pfbad8", 25, [200, 64], [40, 64], page_size=64, num_q_heads=8,
                        num_kv_heads=2, head_dim=128, kv_dtype="e4m3", pool_slack=0.5,
                        chunk_rows=[0, 1])
    st = GpuState(w)
    st.append_step()
    q, cu, table, lens, max_q = st.chunk_inputs()
    table[0, 1] = -1
    out, lse = st.pkv.paged_prefill_chunk_attention(st.cache, q, cu, table, lens, max_q,
                                                    w.softmax_scale)
    torch.cuda.synchronize()
    assert int(st.flags.item()) & 0x1
    assert torch.all(torch.isfinite(out.float()))
    ref, ref_lse = _oracle_prefill(w)
    rows = np.arange(int(cu[1].item()), int(cu[2].item()))
    compare(out, lse, ref, ref_lse, rows=rows)
