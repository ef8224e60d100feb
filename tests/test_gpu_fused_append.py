"""The decode step with the append fused in (``paged_decode_attention_append``).

One launch stores each sequence's new token and attends over all its tokens.
Against the two calls it replaces (``paged_kv_append`` of one token per
sequence, then ``paged_decode_attention``) on the same seeded cache:

* the pools are identical byte for byte, and equal to the oracle's pool;
* out and lse are identical bit for bit (same bytes read, same arithmetic);
* out and lse are within the decode tolerance of the fp64 oracle.

Lengths put the new token at the first and the last slot of a page, in a
sequence of one token, and in long sequences whose last tile a forced small
CTA count leaves to a CTA that holds only part of the sequence.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu

# context lengths before the step: new token at slot 0 of a fresh page (63,
# 127, 255), at the last slot of a page (62, 126), a one-token sequence (0),
# and longer ragged ones
_CTX = [0, 62, 63, 126, 127, 255, 1000, 3000, 4095, 17]


def _pair(w):
    """Two caches built from the same seeds: one for the separate calls, one
    for the fused call."""
    a, b = GpuState(w), GpuState(w)
    torch.cuda.synchronize()
    return a, b


def _run(w, num_ctas=0):
    import paged_kv_cache_476_b200 as pkv

    sep, fus = _pair(w)
    sep.append_step()
    out_s, lse_s = sep.decode(num_ctas=num_ctas)
    q, table, lens, max_len = fus.decode_inputs()
    k_new = fus.k_new.to("cuda").contiguous()
    v_new = fus.v_new.to("cuda").contiguous()
    out_f, lse_f = pkv.paged_decode_attention_append(fus.cache, q, table, lens, max_len, k_new,
                                                     v_new, w.softmax_scale, num_ctas=num_ctas)
    torch.cuda.synchronize()
    return sep, fus, (out_s, lse_s), (out_f, lse_f)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
@pytest.mark.parametrize("P,D,Hq,Hkv", [(64, 128, 32, 8), (128, 128, 64, 8), (64, 64, 8, 8)])
@pytest.mark.parametrize("num_ctas", [0, 3])
def test_fused_equals_append_then_decode(dtype, P, D, Hq, Hkv, num_ctas):
    w = workloads.build("fused", 61, _CTX, [1] * len(_CTX), page_size=P, num_q_heads=Hq,
                        num_kv_heads=Hkv, head_dim=D, kv_dtype=dtype, pool_slack=0.2)
    sep, fus, (out_s, lse_s), (out_f, lse_f) = _run(w, num_ctas)
    ks, vs = sep.pool_bytes()
    kf, vf = fus.pool_bytes()
    assert np.array_equal(ks, kf) and np.array_equal(vs, vf), "pools differ"
    c = oracle.cache_for(w)
    assert np.array_equal(kf, c.k_pool) and np.array_equal(vf, c.v_pool), "pool != oracle"
    assert torch.equal(out_s, out_f), "out differs from the separate calls"
    assert torch.equal(lse_s, lse_f), "lse differs from the separate calls"
    ref, ref_lse = c.decode(oracle.bf16_bits(w.q_decode()), w.page_table, w.lens_after,
                            w.softmax_scale)
    compare(out_f, lse_f, ref, ref_lse)
    assert int(fus.flags.item()) == 0 and int(sep.flags.item()) == 0


def test_fused_llama8b_shaped_batch():
    # the 64-sequence decode batch of the bandwidth benchmark, default plan
    w = workloads.config(2)
    sep, fus, (out_s, lse_s), (out_f, lse_f) = _run(w)
    ks, vs = sep.pool_bytes()
    kf, vf = fus.pool_bytes()
    assert np.array_equal(ks, kf) and np.array_equal(vs, vf)
    assert torch.equal(out_s, out_f) and torch.equal(lse_s, lse_f)
    assert int(fus.flags.item()) == 0


def test_fused_rejects_missing_or_misshaped_tokens():
    import paged_kv_cache_476_b200 as pkv

    w = workloads.config(1)
    st = GpuState(w)
    q, table, lens, max_len = st.decode_inputs()
    k_new = st.k_new.to("cuda").contiguous()
    with pytest.raises(ValueError):
        pkv.paged_decode_attention_append(st.cache, q, table, lens, max_len, k_new[:, :1], k_new)
    lib = pkv.lib()
    out = torch.empty_like(q)
    ws = pkv.decode_workspace(st.cache, q.shape[0], q.shape[1], max_len, 0)
    import ctypes

    st_code = lib.paged_decode_attention_append(
        ctypes.byref(st.cache.c_struct), q.data_ptr(), q.shape[1], q.shape[1] // w.num_kv_heads,
        table.data_ptr(), table.shape[1], lens.data_ptr(), q.shape[0], max_len,
        w.softmax_scale, None, k_new.data_ptr(), out.data_ptr(), None, ws.data_ptr(),
        ws.numel(), 0, None)
    assert st_code == -1  # PKV_ERR_NULL: k_new missing
