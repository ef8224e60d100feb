"""The mixed in-flight step captured in a CUDA graph (needs a GPU).

Append + decode (two kernels joined by a programmatic dependent launch) +
prefill of the mixed configuration are captured once with torch's CUDA-graph
API through the library's binding and replayed.  Every kernel is
deterministic for fixed inputs and launch shapes, so a replay must give the
same bits as the eager step, and both must match the oracle.
"""
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager_step():
    import paged_kv_cache_476_b200 as pkv

    w = workloads.mixed_inflight()
    st = GpuState(w)
    cache = st.cache
    q, table, lens, max_len = st.decode_inputs()
    pq, cu, ptable, plens, max_q = st.chunk_inputs()
    a_lens = torch.from_numpy(w.ctx_lens).cuda()
    a_cu = torch.from_numpy(w.cu_new()).cuda()
    k_new, v_new = st.k_new.cuda(), st.v_new.cuda()
    ws = pkv.decode_workspace(cache, q.shape[0], w.num_q_heads, max_len)
    d_out, d_lse = torch.empty_like(q), torch.empty(q.shape[:2], dtype=torch.float32,
                                                    device=q.device)
    p_out, p_lse = torch.empty_like(pq), torch.empty(pq.shape[:2], dtype=torch.float32,
                                                     device=pq.device)

    def step():  # inputs staged above: nothing but library launches inside
        pkv.paged_kv_append(cache, st.table, a_lens, a_cu, k_new, v_new)
        pkv.paged_decode_attention(cache, q, table, lens, max_len, w.softmax_scale, out=d_out,
                                   lse=d_lse, workspace=ws)
        pkv.paged_prefill_chunk_attention(cache, pq, cu, ptable, plens, max_q, w.softmax_scale,
                                          out=p_out, lse=p_lse)

    step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in (d_out, d_lse, p_out, p_lse)]
    for t in (d_out, d_lse, p_out, p_lse):
        t.fill_(0)

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            step()
    torch.cuda.synchronize()
    for t in (d_out, d_lse, p_out, p_lse):
        t.fill_(0)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager, (d_out, d_lse, p_out, p_lse)):
        assert torch.equal(a, b)
    assert int(st.flags.item()) == 0
    c = oracle.cache_for(w)
    ref, ref_lse = c.decode(oracle.bf16_bits(w.q_decode()), w.page_table[w.decode_rows],
                            w.lens_after[w.decode_rows], w.softmax_scale)
    compare(d_out, d_lse, ref, ref_lse)
    rows = w.chunk_rows
    pref, pref_lse = c.prefill_chunk(oracle.bf16_bits(w.q_chunks()), w.cu_q_chunks(),
                                     w.page_table[rows], w.lens_after[rows], w.softmax_scale)
    compare(p_out, p_lse, pref, pref_lse)
    del g
