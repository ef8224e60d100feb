"""FP4 (NVFP4) KV pools on the GPU against the oracle (needs a GPU).

The pools hold E2M1 codes (two per byte) and an E4M3 block scale per 16
values of a row, after all the codes, with the per-(page, kv head) fp32
scale of the other quantised formats (solosoft post, FAQ: FP4 quantisation
on Blackwell).  The append must write exactly the oracle's bytes (codes,
block scales, and every untouched sentinel byte).  Decode and prefill read
those pools and must match the oracle attending over its own bit-identical
FP4 pool: max-abs 1e-2 (with the output-rounding allowance above |exact| = 2),
mean-abs 1e-3, lse 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare
from tests.test_gpu_append_decode import _check_pool, _oracle_decode
from tests.test_gpu_prefill import _oracle_prefill

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P,D", [(64, 64), (64, 128), (128, 128), (128, 64)])
def test_nvfp4_append_is_bit_exact(P, D):
    w = workloads.build("fp4append", 71, [0, 1, 63, 64, 127, 200, 5], [1, 1, 1, 65, 2, 129, 300],
                        page_size=P, num_q_heads=8, num_kv_heads=2, head_dim=D,
                        kv_dtype="nvfp4", pool_slack=0.25)
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    assert int(st.flags.item()) == 0


def test_nvfp4_append_small_scales_saturate_like_the_oracle():
    # per-page scales far below absmax/(448*6): block scales saturate at 448
    # and codes at +-6, exactly as the oracle's encoder does
    w = workloads.build("fp4sat", 72, [10, 70], [3, 1], page_size=64, num_q_heads=2,
                        num_kv_heads=1, head_dim=128, kv_dtype="nvfp4", pool_slack=0.5)
    st = GpuState(w)
    st.k_scale.fill_(2.0 ** -12)
    st.v_scale.fill_(0.37)
    st.append_step()
    torch.cuda.synchronize()
    c = oracle.cache_for(w, include_new=False)
    c.k_scale[:] = 2.0 ** -12
    c.v_scale[:] = 0.37
    k_new, v_new = w.new_kv()
    c.append(w.page_table, w.ctx_lens, w.cu_new(), oracle.bf16_bits(k_new),
             oracle.bf16_bits(v_new))
    k, v = st.pool_bytes()
    assert np.array_equal(k, c.k_pool) and np.array_equal(v, c.v_pool)
    rows = w.num_pages * w.page_size
    assert (k[rows * 64:] == 0x7E).any()  # a block scale saturated at 448


CASES = [
    # (P, D, Hkv, G, ctx lengths)
    (64, 128, 8, 8, [0, 1, 63, 64, 300, 1500, 4095]),
    (128, 128, 2, 4, [0, 129, 1000, 2047]),
    (64, 64, 2, 2, [3, 64, 65, 400]),
    (128, 64, 1, 1, [255, 256, 1, 2000]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"P{c[0]}-D{c[1]}-G{c[3]}")
@pytest.mark.parametrize("num_ctas", [0, 1, 7])
def test_nvfp4_decode_matches_oracle(case, num_ctas):
    P, D, Hkv, G, ctx = case
    w = workloads.build("fp4dec", 73, ctx, [1] * len(ctx), page_size=P, num_q_heads=Hkv * G,
                        num_kv_heads=Hkv, head_dim=D, kv_dtype="nvfp4", pool_slack=0.3)
    st = GpuState(w)
    st.append_step()
    out, lse = st.decode(num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


PREFILL_CASES = [
    (64, 128, 2, 4, [0, 100, 700], [512, 33, 130]),
    (128, 128, 1, 8, [5, 0, 300], [17, 1, 129]),
    (64, 64, 2, 2, [63, 64, 0], [65, 1, 300]),
    (128, 64, 2, 1, [1000], [200]),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: f"P{c[0]}-D{c[1]}-G{c[3]}")
def test_nvfp4_prefill_matches_oracle(case):
    P, D, Hkv, G, ctx, new = case
    w = workloads.build("fp4pf", 74, ctx, new, page_size=P, num_q_heads=Hkv * G,
                        num_kv_heads=Hkv, head_dim=D, kv_dtype="nvfp4", pool_slack=0.3,
                        chunk_rows=range(len(ctx)))
    st = GpuState(w)
    st.append_step()
    out, lse = st.prefill()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_prefill(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


@pytest.mark.parametrize("P,D,Hq,Hkv", [(64, 128, 32, 8), (128, 64, 8, 8)])
def test_nvfp4_fused_append_equals_append_then_decode(P, D, Hq, Hkv):
    import paged_kv_cache_476_b200 as pkv

    ctx = [0, 62, 63, 126, 127, 255, 1000, 3000, 17]
    w = workloads.build("fp4fused", 75, ctx, [1] * len(ctx), page_size=P, num_q_heads=Hq,
                        num_kv_heads=Hkv, head_dim=D, kv_dtype="nvfp4", pool_slack=0.2)
    sep, fus = GpuState(w), GpuState(w)
    sep.append_step()
    out_s, lse_s = sep.decode()
    q, table, lens, max_len = fus.decode_inputs()
    out_f, lse_f = pkv.paged_decode_attention_append(
        fus.cache, q, table, lens, max_len, fus.k_new.to("cuda").contiguous(),
        fus.v_new.to("cuda").contiguous(), w.softmax_scale)
    torch.cuda.synchronize()
    ks, vs = sep.pool_bytes()
    kf, vf = fus.pool_bytes()
    assert np.array_equal(ks, kf) and np.array_equal(vs, vf)
    _check_pool(fus, w)
    assert torch.equal(out_s, out_f) and torch.equal(lse_s, lse_f)
    ref, ref_lse = _oracle_decode(w)
    compare(out_f, lse_f, ref, ref_lse)


def test_config_70b_nvfp4_decode_full():
    w = workloads.llama70b_nvfp4_decode()
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    out, lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0
