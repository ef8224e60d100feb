"""The kernels' bounded waits give up, report, and leave the GPU usable (needs a GPU).

Every wait inside the library's kernels goes through one helper that stops
after a time limit, ORs PKV_FLAG_TIMEOUT into the caller's error word and
lets the kernel return (the murmur post lists fault recovery among its
evaluation criteria).  ``pkv_check_bounded_wait`` runs that helper on an
mbarrier nothing arrives on, with nothing else in flight.  The failure is
made by a flag that nothing sets: no fault, trap or hang.  Afterwards an
ordinary decode must still run and match the oracle.
"""
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ns", [1_000_000, 0])  # 1 ms, and the kernels' own 2 s
def test_bounded_wait_gives_up_and_reports(limit_ns):
    import paged_kv_cache_476_b200 as pkv

    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    pkv.pkv_check_bounded_wait(flags, limit_ns, waited)
    torch.cuda.synchronize()  # the call returns: the wait ended by itself
    assert int(flags.item()) == pkv.PKV_FLAG_TIMEOUT
    lim = limit_ns or 2_000_000_000
    w_ns = int(waited.item())
    assert lim <= w_ns < lim + 200_000_000, w_ns


def test_gpu_still_answers_after_a_timeout():
    import paged_kv_cache_476_b200 as pkv

    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.pkv_check_bounded_wait(flags, 1_000_000)
    w = workloads.build("after_timeout", 41, [90, 700, 3], [1] * 3, page_size=64,
                        num_q_heads=8, num_kv_heads=2, head_dim=128, pool_slack=0.3)
    st = GpuState(w)  # same stream: runs after the timed-out kernel
    st.append_step()
    out, lse = st.decode()
    torch.cuda.synchronize()
    assert int(flags.item()) == pkv.PKV_FLAG_TIMEOUT
    assert int(st.flags.item()) == 0  # the decode's own waits all completed
    c = oracle.cache_for(w)
    rows = w.decode_rows
    ref, ref_lse = c.decode(oracle.bf16_bits(w.q_decode()), w.page_table[rows],
                            w.lens_after[rows], w.softmax_scale)
    compare(out, lse, ref, ref_lse)
