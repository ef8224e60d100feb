"""Decode work split on batches of short units, against the oracle (needs a GPU).

For quantised pools the decode splits its work list in virtual tiles: each
(sequence, kv head) unit counts its tiles plus one tile that loads nothing and
stands for the cost of a unit end.  With many one- to three-tile units and a
CTA count near the virtual total, ranges start, end and sit entirely on those
end costs (a range may then hold no real tile at all), and units are cut at
every kind of boundary.  Every such split must still give the oracle's
attention: max-abs 1e-2 (with the output-rounding allowance above |exact| =
2), mean-abs 1e-3, lse 2e-3, and no error flag.  bf16 pools (no end cost) run
the same sweep.
"""
import pytest
import torch

import workloads
from tests._gpu import GpuState, compare
from tests.test_gpu_append_decode import _oracle_decode

pytestmark = pytest.mark.gpu

# context lengths before the appended token: one to three 128-token tiles
# (one to five 64-token tiles) per unit, one empty context
CTX = [0, 1, 5, 127, 128, 129, 200, 255, 256, 300, 3, 64]


@pytest.mark.parametrize("dtype", ["e4m3", "int8", "nvfp4", "bf16"])
@pytest.mark.parametrize("num_ctas", [1, 2, 3, 5, 8, 13, 21, 31, 32, 33, 47, 63, 64, 65, 5000])
def test_decode_split_over_short_units(dtype, num_ctas):
    w = workloads.build("split", 81, CTX, [1] * len(CTX), page_size=64, num_q_heads=8,
                        num_kv_heads=2, head_dim=128, kv_dtype=dtype, pool_slack=0.3)
    st = GpuState(w)
    st.append_step()
    out, lse = st.decode(num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


@pytest.mark.parametrize("dtype", ["e4m3", "int8"])
def test_decode_split_mixed_long_and_short_units(dtype):
    # long units cut across many CTAs next to runs of one-tile units
    ctx = [4000, 1, 2, 3, 130, 1, 2900, 5, 6, 7, 8, 255, 3100, 0]
    w = workloads.build("split2", 82, ctx, [1] * len(ctx), page_size=64, num_q_heads=16,
                        num_kv_heads=2, head_dim=128, kv_dtype=dtype, pool_slack=0.2)
    st = GpuState(w)
    st.append_step()
    for num_ctas in (0, 9, 40, 111):
        out, lse = st.decode(num_ctas=num_ctas)
        torch.cuda.synchronize()
        ref, ref_lse = _oracle_decode(w)
        compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0
