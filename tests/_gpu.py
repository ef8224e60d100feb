"""GPU-side fixtures: build a workload's paged pool through the library's own
append kernel, and compare library results with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import workloads


def sentinel_pool(w, device):
    shape = w.pool_shape()
    if w.kv_dtype == "nvfp4":  # one flat buffer: codes, then block scales
        return torch.full((w.pool_bytes(),), workloads.sentinel_byte(w.kv_dtype),
                          dtype=torch.uint8, device=device)
    if w.kv_dtype != "bf16":
        return torch.full(shape, workloads.sentinel_byte(w.kv_dtype), dtype=torch.uint8,
                          device=device)
    return torch.full(shape, workloads.BF16_NAN_BITS, dtype=torch.int16,
                      device=device).view(torch.bfloat16)


class GpuState:
    """Device pool of workload ``w``: context tokens appended, step tokens pending."""

    def __init__(self, w, device="cuda", group_tokens=1 << 19):
        import paged_kv_cache_476_b200 as pkv

        self.pkv = pkv
        self.w = w
        self.device = device
        self.k_pool = sentinel_pool(w, device)
        self.v_pool = sentinel_pool(w, device)
        self.flags = torch.zeros(1, dtype=torch.int32, device=device)
        self.k_scale = self.v_scale = None
        if w.kv_dtype != "bf16":
            self.k_scale = torch.ones((w.num_pages, w.num_kv_heads), dtype=torch.float32,
                                      device=device)
            self.v_scale = torch.ones_like(self.k_scale)
        self.cache = pkv.PagedKVCache(self.k_pool, self.v_pool, w.kv_dtype, self.k_scale,
                                      self.v_scale, self.flags,
                                      geometry=w.pool_shape() if w.kv_dtype == "nvfp4" else None)
        self.table = torch.from_numpy(w.page_table).to(device)
        self.k_new, self.v_new = [], []
        # Context, in groups of sequences, through the library's append.
        group, n = [], 0
        for b in range(w.batch):
            group.append(b)
            n += int(w.ctx_lens[b])
            if n >= group_tokens or b == w.batch - 1:
                self._append_context(group)
                group, n = [], 0
        self.k_new = torch.cat(self.k_new) if self.k_new else None
        self.v_new = torch.cat(self.v_new) if self.v_new else None
        torch.cuda.synchronize()

    def _append_context(self, rows):
        w = self.w
        ks, vs, cu = [], [], [0]
        for b in rows:
            k, v = w.kv_seq(b)
            c = int(w.ctx_lens[b])
            if w.kv_dtype != "bf16":
                pages, k_s, v_s = w.kv_scales_for(b, k, v)
                idx = torch.from_numpy(pages.astype(np.int64)).to(self.device)
                self.k_scale[idx] = torch.from_numpy(k_s).to(self.device)
                self.v_scale[idx] = torch.from_numpy(v_s).to(self.device)
            ks.append(k[:c])
            vs.append(v[:c])
            cu.append(cu[-1] + c)
            self.k_new.append(k[c:])
            self.v_new.append(v[c:])
        if cu[-1] == 0:
            return
        rows_t = torch.tensor(rows, dtype=torch.long, device=self.device)
        table = self.table[rows_t].contiguous()
        zeros = torch.zeros(len(rows), dtype=torch.int32, device=self.device)
        cu_t = torch.tensor(cu, dtype=torch.int32, device=self.device)
        k = torch.cat(ks).to(self.device)
        v = torch.cat(vs).to(self.device)
        self.pkv.paged_kv_append(self.cache, table, zeros, cu_t, k, v)

    def append_step(self):
        """Append this step's new tokens of every sequence in one call."""
        w = self.w
        lens = torch.from_numpy(w.ctx_lens).to(self.device)
        cu = torch.from_numpy(w.cu_new()).to(self.device)
        self.pkv.paged_kv_append(self.cache, self.table, lens, cu, self.k_new.to(self.device),
                                 self.v_new.to(self.device))

    def decode_inputs(self):
        w = self.w
        rows = torch.from_numpy(w.decode_rows).to(self.device)
        q = w.q_decode().to(self.device)
        table = self.table[rows].contiguous()
        lens = torch.from_numpy(w.lens_after[w.decode_rows]).to(self.device)
        max_len = int(w.lens_after[w.decode_rows].max()) if len(w.decode_rows) else 0
        return q, table, lens, max_len

    def decode(self, num_ctas=0):
        q, table, lens, max_len = self.decode_inputs()
        return self.pkv.paged_decode_attention(self.cache, q, table, lens, max_len,
                                               self.w.softmax_scale, num_ctas=num_ctas)

    def chunk_inputs(self):
        w = self.w
        rows = torch.from_numpy(w.chunk_rows).to(self.device)
        q = w.q_chunks().to(self.device)
        table = self.table[rows].contiguous()
        lens = torch.from_numpy(w.lens_after[w.chunk_rows]).to(self.device)
        cu = torch.from_numpy(w.cu_q_chunks()).to(self.device)
        max_q = int(w.new_lens[w.chunk_rows].max()) if len(w.chunk_rows) else 0
        return q, cu, table, lens, max_q

    def prefill(self):
        q, cu, table, lens, max_q = self.chunk_inputs()
        return self.pkv.paged_prefill_chunk_attention(self.cache, q, cu, table, lens, max_q,
                                                      self.w.softmax_scale)

    def pool_bytes(self):
        return (self.k_pool.view(torch.uint8).cpu().numpy().reshape(-1),
                self.v_pool.view(torch.uint8).cpu().numpy().reshape(-1))


def bf16_half_ulp(x):
    """Half the bf16 spacing at |x| (8 significant bits): what rounding the exact
    value to bf16 may cost at best."""
    _, e = np.frexp(np.abs(x))  # |x| = m * 2^e, m in [0.5, 1)
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def bf16_round(x):
    """fp64 values rounded to the nearest bf16 (8 significant bits), ties to
    even: the correctly rounded bf16 answer of an exact value."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, |m| in [0.5, 1)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


# Elements that met the bound only through its rounding allowance, per
# compare() call (a record for the test log).
ROUNDED_ONLY = []


def compare(out, lse, ref_out, ref_lse, rows=None, max_abs=1e-2, mean_abs=1e-3, lse_abs=2e-3):
    """bf16 output vs fp64 oracle; fp32 lse bound.

    Every element must satisfy |out - exact| <= max_abs, with one narrow
    allowance for the output's own rounding to bf16: where |exact| >= 2 (half
    a bf16 ulp is then at least 2^-8, over a third of max_abs), an element
    may instead be the correctly rounded bf16 value of some number within
    max_abs of the exact result, i.e. |out - exact| <= max_abs + half an ulp
    of out.  The allowance never applies below |exact| = 2; the number of
    elements that needed it is printed and recorded in ROUNDED_ONLY.  The
    mean of |out - exact| must stay <= mean_abs.
    """
    o = out.float().cpu().numpy().astype(np.float64)
    r = ref_out
    if rows is not None:
        o, r = o[rows], r[rows]
    assert np.all(np.isfinite(o)), "non-finite output"
    err = np.abs(o - r)
    plain = err <= max_abs
    allowed = ~plain & (np.abs(r) >= 2.0) & (err <= max_abs + bf16_half_ulp(o))
    bad = ~plain & ~allowed
    info = (f"max_abs={err.max():.3e} mean_abs={err.mean():.3e} "
            f"elements over the bound: {int(bad.sum())}"
            + (f" (worst at exact={r[bad][np.argmax(err[bad])]:.6f}, "
               f"out={o[bad][np.argmax(err[bad])]:.6f})" if bad.any() else ""))
    assert not bad.any(), info
    n_allowed = int(allowed.sum())
    if n_allowed:
        exact_rounded = int((o[allowed] == bf16_round(r[allowed])).sum())
        print(f"compare: {n_allowed} of {err.size} elements over {max_abs} only by the output's "
              f"rounding (|exact| >= 2; {exact_rounded} of them the correctly rounded value; "
              f"worst |out - exact| {err[allowed].max():.4e})")
    ROUNDED_ONLY.append(n_allowed)
    assert err.mean() <= mean_abs, info
    if lse is not None and ref_lse is not None:
        l = lse.cpu().numpy().astype(np.float64)
        rl = ref_lse
        if rows is not None:
            l, rl = l[rows], rl[rows]
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(l), fin)
        if fin.any():
            le = np.abs(l[fin] - rl[fin]).max()
            assert le <= lse_abs, f"lse err {le:.3e}"
    return err.max(), err.mean()
