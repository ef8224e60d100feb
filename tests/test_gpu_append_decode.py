"""Parity of the CUDA append and decode kernels with the oracle (needs a GPU).

Append: the device pool must equal the oracle's own pool byte for byte (bf16
bits, E4M3 or INT8 codes, and every untouched sentinel byte).  Decode: bf16 output
within max-abs 1e-2 and mean-abs 1e-3 of the fp64 oracle; lse within 2e-3.
Inputs are the seeded synthetic workloads (shapes of the five benchmark
configurations plus ragged edge cases).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests._gpu import GpuState, compare

pytestmark = pytest.mark.gpu


def _oracle_decode(w, seq_ids=None):
    c = oracle.cache_for(w, seq_ids=seq_ids)
    q = oracle.bf16_bits(w.q_decode())
    rows = w.decode_rows
    ids = None if seq_ids is None else [int(np.nonzero(rows == b)[0][0]) for b in seq_ids]
    return c.decode(q, w.page_table[rows], w.lens_after[rows], w.softmax_scale, seq_ids=ids)


def _check_pool(st, w):
    c = oracle.cache_for(w)
    k, v = st.pool_bytes()
    assert np.array_equal(k, c.k_pool), "K pool differs from the oracle's"
    assert np.array_equal(v, c.v_pool), "V pool differs from the oracle's"


# ------------------------------------------------------------------ append
@pytest.mark.parametrize("dtype", ["bf16", "e4m3", "int8"])
@pytest.mark.parametrize("P,D", [(64, 64), (64, 128), (128, 128), (128, 64)])
def test_append_is_bit_exact(dtype, P, D):
    w = workloads.build("append", 7, [0, 1, 63, 64, 127, 200, 5], [1, 1, 1, 65, 2, 129, 300],
                        page_size=P, num_q_heads=8, num_kv_heads=2, head_dim=D,
                        kv_dtype=dtype, pool_slack=0.25)
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    assert int(st.flags.item()) == 0


def test_append_e4m3_saturates_like_the_oracle():
    # scales far below absmax/448: most values saturate to +-448
    w = workloads.build("sat", 8, [10, 70], [3, 1], page_size=64, num_q_heads=2,
                        num_kv_heads=1, head_dim=128, kv_dtype="e4m3", pool_slack=0.5)
    st = GpuState(w)
    st.k_scale.fill_(2.0**-9)
    st.v_scale.fill_(0.37)
    st.append_step()
    torch.cuda.synchronize()
    c = oracle.Cache(w.num_pages, 64, 1, 128, "e4m3",
                     np.full(w.pool_bytes(), workloads.E4M3_NAN_CODE, np.uint8),
                     np.full(w.pool_bytes(), workloads.E4M3_NAN_CODE, np.uint8),
                     np.full((w.num_pages, 1), 2.0**-9, np.float32),
                     np.full((w.num_pages, 1), 0.37, np.float32))
    # the oracle's pool: context under the fill-time scales, then the step
    # tokens under the new scales -- rebuild the context the same way
    ref = oracle.cache_for(w, include_new=False)
    c.k_pool[:] = ref.k_pool
    c.v_pool[:] = ref.v_pool
    k_new, v_new = w.new_kv()
    c.append(w.page_table, w.ctx_lens, w.cu_new(), oracle.bf16_bits(k_new),
             oracle.bf16_bits(v_new))
    k, v = st.pool_bytes()
    assert np.array_equal(k, c.k_pool) and np.array_equal(v, c.v_pool)
    assert (k == 0x7E).any() and (k == 0xFE).any()


def test_append_int8_clamps_like_the_oracle():
    # scales far below absmax/127: most codes clamp to +-127 (never -128)
    w = workloads.build("sat8", 8, [10, 70], [3, 1], page_size=64, num_q_heads=2,
                        num_kv_heads=1, head_dim=128, kv_dtype="int8", pool_slack=0.5)
    st = GpuState(w)
    st.k_scale.fill_(2.0**-9)
    st.v_scale.fill_(0.013)
    st.append_step()
    torch.cuda.synchronize()
    c = oracle.cache_for(w, include_new=False)
    c.k_scale[:] = 2.0**-9
    c.v_scale[:] = 0.013
    k_new, v_new = w.new_kv()
    c.append(w.page_table, w.ctx_lens, w.cu_new(), oracle.bf16_bits(k_new),
             oracle.bf16_bits(v_new))
    k, v = st.pool_bytes()
    assert np.array_equal(k, c.k_pool) and np.array_equal(v, c.v_pool)
    new_k = k.view(np.int8)
    assert (new_k == 127).any() and (new_k == -127).any()


def test_append_bad_page_is_skipped_and_flagged():
    w = workloads.build("bad", 9, [3, 3], [1, 1], page_size=64, num_q_heads=2, num_kv_heads=1,
                        head_dim=64, pool_slack=1.0)
    st = GpuState(w)
    st.table[1, 0] = w.num_pages + 5  # out of range: sequence 1's token must not land
    st.append_step()
    torch.cuda.synchronize()
    assert int(st.flags.item()) & 0x1
    ref = oracle.cache_for(w, include_new=False)
    k_new, v_new = w.new_kv(rows=[0])
    ref.append(w.page_table[:1], w.ctx_lens[:1], [0, 1], oracle.bf16_bits(k_new),
               oracle.bf16_bits(v_new))
    k, v = st.pool_bytes()
    assert np.array_equal(k, ref.k_pool) and np.array_equal(v, ref.v_pool)


# ------------------------------------------------------------------ decode
def test_tiny_config_append_and_decode():
    w = workloads.tiny_decode()
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    out, lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


CASES = [
    # (dtype, P, D, Hkv, G, ctx lengths)
    ("bf16", 64, 128, 8, 4, [0, 1, 62, 63, 64, 127, 128, 500, 1000, 4000]),
    ("bf16", 128, 128, 2, 8, [0, 5, 127, 128, 129, 1023, 3000]),
    ("bf16", 64, 64, 4, 1, [0, 17, 64, 100, 130, 700]),
    ("bf16", 128, 64, 1, 2, [255, 256, 1, 2000]),
    ("e4m3", 64, 128, 8, 8, [0, 1, 63, 64, 300, 1500, 4095]),
    ("e4m3", 128, 128, 2, 4, [0, 129, 1000, 2047]),
    ("e4m3", 64, 64, 2, 2, [3, 64, 65, 400]),
    ("int8", 64, 128, 8, 8, [0, 1, 63, 64, 300, 1500, 4095]),
    ("int8", 128, 128, 2, 4, [0, 129, 1000, 2047]),
    ("int8", 64, 64, 2, 1, [3, 64, 65, 400]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-P{c[1]}-D{c[2]}-G{c[4]}")
@pytest.mark.parametrize("num_ctas", [0, 1, 7, 5000])
def test_decode_matches_oracle(case, num_ctas):
    dtype, P, D, Hkv, G, ctx = case
    w = workloads.build("dec", 11, ctx, [1] * len(ctx), page_size=P, num_q_heads=Hkv * G,
                        num_kv_heads=Hkv, head_dim=D, kv_dtype=dtype, pool_slack=0.3)
    st = GpuState(w)
    st.append_step()
    out, lse = st.decode(num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


def test_decode_is_deterministic_at_fixed_ctas_and_close_across():
    w = workloads.build("det", 12, [3000, 40, 900, 2500], [1] * 4, page_size=64,
                        num_q_heads=32, num_kv_heads=8, head_dim=128, pool_slack=0.1)
    st = GpuState(w)
    st.append_step()
    a, la = st.decode(num_ctas=5)
    b, lb = st.decode(num_ctas=5)
    c, lc = st.decode(num_ctas=300)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert (a.float() - c.float()).abs().max().item() <= 1.6e-2


def test_decode_empty_sequence_gives_zero_and_minus_inf():
    w = workloads.build("empty", 13, [0, 70, 0], [0, 1, 0], page_size=64, num_q_heads=4,
                        num_kv_heads=1, head_dim=128, pool_pages=4)
    st = GpuState(w)
    st.append_step()
    out, lse = st.decode()
    torch.cuda.synchronize()
    o = out.float().cpu()
    assert torch.all(o[0] == 0) and torch.all(o[2] == 0)
    assert torch.all(torch.isneginf(lse[0].cpu())) and torch.all(torch.isneginf(lse[2].cpu()))
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse, rows=[1])


def test_decode_bad_page_is_masked_and_flagged():
    w = workloads.build("badp", 14, [200, 300], [1, 1], page_size=64, num_q_heads=8,
                        num_kv_heads=2, head_dim=128, pool_slack=0.5)
    st = GpuState(w)
    st.append_step()
    q, table, lens, max_len = st.decode_inputs()
    table[0, 1] = -7
    out, lse = st.pkv.paged_decode_attention(st.cache, q, table, lens, max_len, w.softmax_scale)
    torch.cuda.synchronize()
    assert int(st.flags.item()) & 0x1
    assert torch.all(torch.isfinite(out.float()))
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse, rows=[1])


# ---------------------------------------------- the benchmark configurations
def test_config_llama8b_decode_full():
    w = workloads.llama8b_decode()
    st = GpuState(w)
    st.append_step()
    out, lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


def test_config_long_context_decode_full():
    # all 8 sequences (32k-131k tokens each) against the oracle
    w = workloads.long_context_decode()
    st = GpuState(w)
    st.append_step()
    out, lse = st.decode()
    torch.cuda.synchronize()
    assert int(st.flags.item()) == 0
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)


def test_config_70b_fp8_decode_full():
    w = workloads.llama70b_fp8_decode()
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    out, lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


def test_config_70b_int8_decode_full():
    w = workloads.llama70b_int8_decode()
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    out, lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)
    assert int(st.flags.item()) == 0


def test_config_mixed_decode_part():
    w = workloads.mixed_inflight()
    st = GpuState(w)
    st.append_step()
    torch.cuda.synchronize()
    _check_pool(st, w)
    out, lse = st.decode()
    torch.cuda.synchronize()
    ref, ref_lse = _oracle_decode(w)
    compare(out, lse, ref, ref_lse)


def test_workspace_reused_across_batch_shapes():
    # one workspace serves calls with other shapes after it: each call writes
    # every workspace value it reads, so the previous call's contents are harmless
    import paged_kv_cache_476_b200 as pkv

    big = workloads.build("wsA", 15, [3000, 9000, 40, 2500] * 8, [1] * 32, page_size=64,
                          num_q_heads=32, num_kv_heads=8, head_dim=128, pool_slack=0.1)
    small = workloads.build("wsB", 16, [700, 5, 1500], [1] * 3, page_size=64,
                            num_q_heads=16, num_kv_heads=2, head_dim=128, pool_slack=0.2)
    need = max(pkv.paged_decode_workspace_bytes(32, 32, 8, 128, 9001),
               pkv.paged_decode_workspace_bytes(3, 16, 2, 128, 1501))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for w in (big, small, big, small):
        st = GpuState(w)
        st.append_step()
        q, table, lens, max_len = st.decode_inputs()
        out, lse = pkv.paged_decode_attention(st.cache, q, table, lens, max_len, w.softmax_scale,
                                              workspace=ws)
        torch.cuda.synchronize()
        ref, ref_lse = _oracle_decode(w)
        compare(out, lse, ref, ref_lse)
