#!/usr/bin/env python
"""Benchmark: paged-KV decode step (append + split-KV decode) on B200.

One step = the whole hot path over one batch: append this step's new K/V
through the page table, then decode attention over every cached token (and,
for the in-flight mixed batch, the causal prefill chunks).  The headline
workload is the Llama-3-8B-shaped batch (64 sequences, context U[128,4096],
page size 64, 32 q / 8 kv heads, head_dim 128, bf16).  Inputs are seeded
synthetic data resident in HBM; the KV pool (~0.6 GB) exceeds the 126 MB L2,
so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..6]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Prints ONE JSON line (rank 0).  ``value`` is whole-job achieved HBM GB/s of
algorithmic bytes (K/V + scales + Q/out + page-table entries + appended
rows) per step time; tokens/s is reported beside it.  At N = 1 the line
also carries ``per_config``: every workload shape (tiny, 8B-shaped, long
context, 70B-shaped E4M3 and INT8, in-flight mixed) with its step time, each
kernel's time alone, its roofline and the parity of its outputs against the
oracle on a bounded sample.  Multi-GPU runs are weak scaling: each rank runs
its own batch, no data-path collective.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-KV decode attention: achieved HBM GB/s (% of B200 peak), tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
# Each graph-replayed kernel measurement spans at least this long, so that
# the clock sampler (every 2 ms) sees it under load many times.
MIN_REGION_S = 0.06
# Soak of the step graph before the headline timed region (clocks settle and
# the sampler runs through it into the timed steps).
SOAK_S = 0.25


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--per-config", default="1,2,3,4,5,6,7",
                    help="workloads measured into per_config at N = 1 ('' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seqs", type=int, default=64)
    return ap.parse_args()


def max_over_ranks(x: float, dist, device=None) -> float:
    """Largest value of ``x`` over all ranks (identity without a process group).

    Multi-GPU times are the max over ranks, taken on the device tensors of
    the rank (NCCL) or on CPU tensors (gloo).
    """
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Weak-scaling throughput: units all ranks processed / the slowest rank's time."""
    return world * units_per_rank / seconds


def profile_traffic(name: str, sources):
    """ncu DRAM bytes per call from ``profiles/<name>``, if the sources still match.

    The kernel's sources are hashed; a capture taken on other sources is
    stale and reported as null.
    """
    import hashlib

    src = os.path.join(ROOT, "paged_kv_cache_476_b200", "csrc")
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(src, f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:16]
    try:
        with open(os.path.join(ROOT, "profiles", name)) as fh:
            kv = dict(line.strip().split(": ", 1) for line in fh if ": " in line and
                      line.startswith(("traffic_bytes_per_call", "source_sha256_16")))
        if kv.get("source_sha256_16") == sha:
            return int(kv["traffic_bytes_per_call"])
    except (OSError, ValueError, KeyError):
        pass
    return None


DECODE_SOURCES = ("decode.cu", "common.cuh", "kernels.h")
PREFILL_SOURCES = ("prefill.cu", "common.cuh", "kernels.h")
# ncu summaries whose per-call DRAM traffic feeds the roofline, by workload
TRAFFIC_PROFILES = {
    2: ("decode", "decode_kernel_llama8b_decode.md", DECODE_SOURCES),
    4: ("decode", "decode_kernel_llama70b_e4m3.md", DECODE_SOURCES),
    6: ("decode", "decode_kernel_llama70b_int8.md", DECODE_SOURCES),
    7: ("decode", "decode_kernel_llama70b_nvfp4.md", DECODE_SOURCES),
}


def peaks():
    """(hbm GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def decode_roofline(dec_s, dec_bytes, hbm_peak, peak_kind, traffic=None):
    """Decode (HBM-bound): algorithmic bytes / its time against the measured copy bandwidth."""
    achieved = dec_bytes / dec_s / 1e9
    return {
        "bound": "hbm",
        "kernel": "decode_kernel + decode_merge_kernel (one paged_decode_attention call)",
        "achieved": round(achieved, 1),
        "peak": hbm_peak,
        "unit": "GB/s",
        "frac": round(achieved / hbm_peak, 4),
        "peak_source": f"{peak_kind} hbm_gbs (copy bandwidth, burst)",
        "traffic": traffic,
        "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one "
                          "decode_kernel launch (profiles/), null if the sources changed",
        "algorithmic_bytes_per_launch": int(dec_bytes),
    }


def prefill_roofline(pf_s, pf_flops, tf_peak, peak_kind):
    """Prefill (tensor-bound): causal-pair flops / its time against the measured
    burst bf16 GEMM rate (the call is timed alone, graph-replayed)."""
    achieved = pf_flops / pf_s / 1e12
    return {
        "bound": "tensor",
        "kernel": "prefill_kernel (one paged_prefill_chunk_attention call)",
        "achieved": round(achieved, 1),
        "peak": tf_peak,
        "unit": "TFLOP/s",
        "frac": round(achieved / tf_peak, 4),
        "peak_source": f"{peak_kind} bf16_tflops (cuBLAS bf16 GEMM, burst)",
        "traffic": None,
        "traffic_source": "tensor-bound: DRAM traffic not used for the fraction",
        "algorithmic_flops_per_launch": int(pf_flops),
    }


def roofline_of(dec_s, dec_bytes, pf_s, pf_flops, hbm_peak, tf_peak, peak_kind,
                traffic=None):
    """The roofline object of the step's dominant kernel: the prefill call where
    it takes longer than the decode call, else the decode call."""
    if pf_s and pf_flops and pf_s > dec_s:
        return prefill_roofline(pf_s, pf_flops, tf_peak, peak_kind)
    return decode_roofline(dec_s, dec_bytes, hbm_peak, peak_kind, traffic)


# ------------------------------------------------------------ byte counts
def decode_bytes(w, rows=None) -> int:
    """Algorithmic bytes of decode over sequences ``rows`` (default: decode rows)."""
    rows = w.decode_rows if rows is None else np.asarray(rows)
    la = w.lens_after[rows].astype(np.int64)
    P = w.page_size
    pages = int(((la + P - 1) // P).sum())
    if w.kv_dtype == "nvfp4":  # codes (D/2 bytes) + E4M3 block scales (D/16) per row
        kv = int(la.sum()) * w.num_kv_heads * 2 * (w.head_dim // 2 + w.head_dim // 16)
    else:
        kv = int(la.sum()) * w.num_kv_heads * w.head_dim * 2 * w.elem_bytes
    scales = pages * w.num_kv_heads * 2 * 4 if w.kv_dtype != "bf16" else 0
    qo = 2 * len(rows) * w.num_q_heads * w.head_dim * 2
    return kv + scales + qo + pages * 4


def append_bytes(w, rows=None) -> int:
    """Algorithmic bytes of the append over sequences ``rows`` (default: all)."""
    t = int(w.new_lens.sum() if rows is None else w.new_lens[np.asarray(rows)].sum())
    if w.kv_dtype == "nvfp4":  # bf16 in, codes + block scales out, for K and V
        return t * w.num_kv_heads * 2 * (w.head_dim * 2 + w.head_dim // 2 + w.head_dim // 16)
    return t * w.num_kv_heads * w.head_dim * 2 * (2 + w.elem_bytes)


def prefill_flops(w) -> int:
    tot = 0
    for b in w.chunk_rows:
        L, n = int(w.lens_after[b]), int(w.new_lens[b])
        tot += sum(L - n + i + 1 for i in range(n))
    return 4 * w.num_q_heads * w.head_dim * tot


def config_dict(w, world: int) -> dict:
    """The ``config`` object of the JSON line (both arms print the same one)."""
    return {
        "workload": w.name,
        "batch": int(len(w.decode_rows)),
        "prefill_chunks": int(len(w.chunk_rows)),
        "page_size": w.page_size,
        "heads_q_kv": [w.num_q_heads, w.num_kv_heads],
        "head_dim": w.head_dim,
        "kv_dtype": w.kv_dtype,
        "kv_tokens": int(w.decode_kv_tokens()),
        "step_bytes": int(decode_bytes(w) + append_bytes(w)),
        "parallelism": f"dp{world} (independent batches)",
        "l2": f"KV pool {w.pool_bytes() * 2 / 1e6:.0f} MB vs 126 MB L2; no flush",
        "seed": w.seed,
    }


# ------------------------------------------------------------ clock sampler
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nvml:
            self.t.join()

    def summary(self, what: str):
        base = {"sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "window": what}
        base["sm_mhz"] = statistics.median(self.samples) if self.samples else None
        return base


# ------------------------------------------------------------------ setup
def setup_device_state(w, device):
    """Pool filled through the library's own append (context tokens)."""
    import torch
    import paged_kv_cache_476_b200 as pkv
    import workloads

    shape = w.pool_shape()
    if w.kv_dtype != "bf16":
        fill = workloads.sentinel_byte(w.kv_dtype)
        k_pool = torch.full((w.pool_bytes(),), fill, dtype=torch.uint8, device=device)
        v_pool = torch.full((w.pool_bytes(),), fill, dtype=torch.uint8, device=device)
        if w.kv_dtype != "nvfp4":
            k_pool, v_pool = k_pool.view(shape), v_pool.view(shape)
        k_scale = torch.ones((w.num_pages, w.num_kv_heads), dtype=torch.float32, device=device)
        v_scale = torch.ones_like(k_scale)
    else:
        k_pool = torch.full(shape, workloads.BF16_NAN_BITS, dtype=torch.int16,
                            device=device).view(torch.bfloat16)
        v_pool = torch.full(shape, workloads.BF16_NAN_BITS, dtype=torch.int16,
                            device=device).view(torch.bfloat16)
        k_scale = v_scale = None
    flags = torch.zeros(1, dtype=torch.int32, device=device)
    cache = pkv.PagedKVCache(k_pool, v_pool, w.kv_dtype, k_scale, v_scale, flags,
                             geometry=shape if w.kv_dtype == "nvfp4" else None)
    table = torch.from_numpy(w.page_table).to(device)
    k_new, v_new = [], []
    for b in range(w.batch):
        k, v = w.kv_seq(b)
        c = int(w.ctx_lens[b])
        if w.kv_dtype != "bf16":
            pages, ks, vs = w.kv_scales_for(b, k, v)
            idx = torch.from_numpy(pages.astype(np.int64)).to(device)
            k_scale[idx] = torch.from_numpy(ks).to(device)
            v_scale[idx] = torch.from_numpy(vs).to(device)
        if c:
            pkv.paged_kv_append(cache, table[b:b + 1].contiguous(),
                                torch.zeros(1, dtype=torch.int32, device=device),
                                torch.tensor([0, c], dtype=torch.int32, device=device),
                                k[:c].to(device), v[:c].to(device))
        k_new.append(k[c:])
        v_new.append(v[c:])
    torch.cuda.synchronize()
    st = {
        "cache": cache, "flags": flags, "table": table,
        "ctx_lens": torch.from_numpy(w.ctx_lens).to(device),
        "cu_new": torch.from_numpy(w.cu_new()).to(device),
        "k_new": torch.cat(k_new).to(device), "v_new": torch.cat(v_new).to(device),
    }
    rows = torch.from_numpy(w.decode_rows).to(device)
    st["dec_q"] = w.q_decode().to(device)
    st["dec_table"] = table[rows].contiguous()
    st["dec_lens"] = torch.from_numpy(w.lens_after[w.decode_rows]).to(device)
    st["dec_max"] = int(w.lens_after[w.decode_rows].max()) if len(w.decode_rows) else 0
    st["dec_out"] = torch.empty_like(st["dec_q"])
    st["dec_lse"] = torch.empty(st["dec_q"].shape[:2], dtype=torch.float32, device=device)
    if len(w.chunk_rows):
        crow = torch.from_numpy(w.chunk_rows).to(device)
        st["pf_q"] = w.q_chunks().to(device)
        st["pf_table"] = table[crow].contiguous()
        st["pf_lens"] = torch.from_numpy(w.lens_after[w.chunk_rows]).to(device)
        st["pf_cu"] = torch.from_numpy(w.cu_q_chunks()).to(device)
        st["pf_max"] = int(w.new_lens[w.chunk_rows].max())
        st["pf_out"] = torch.empty_like(st["pf_q"])
        st["pf_lse"] = torch.empty(st["pf_q"].shape[:2], dtype=torch.float32, device=device)
    return st


class Runner:
    """The step's library calls on one workload's device state, and graph-replayed
    timing of the whole step or of one call alone."""

    def __init__(self, w, st, num_ctas, device):
        import torch
        import paged_kv_cache_476_b200 as pkv

        self.torch, self.pkv = torch, pkv
        self.w, self.st, self.num_ctas, self.device = w, st, num_ctas, device
        self.has_dec = len(w.decode_rows) > 0
        self.has_pf = len(w.chunk_rows) > 0
        self.ws = pkv.decode_workspace(st["cache"], len(w.decode_rows), w.num_q_heads,
                                       st["dec_max"], num_ctas) if self.has_dec else None
        self.stream = torch.cuda.current_stream()
        self.gstream = torch.cuda.Stream()

    def append(self):
        st = self.st
        self.pkv.paged_kv_append(st["cache"], st["table"], st["ctx_lens"], st["cu_new"],
                                 st["k_new"], st["v_new"])

    def decode(self):
        st, w = self.st, self.w
        if self.has_dec:
            self.pkv.paged_decode_attention(st["cache"], st["dec_q"], st["dec_table"],
                                            st["dec_lens"], st["dec_max"], w.softmax_scale,
                                            out=st["dec_out"], lse=st["dec_lse"],
                                            workspace=self.ws, num_ctas=self.num_ctas)

    def prefill(self):
        st, w = self.st, self.w
        if self.has_pf:
            self.pkv.paged_prefill_chunk_attention(st["cache"], st["pf_q"], st["pf_cu"],
                                                   st["pf_table"], st["pf_lens"], st["pf_max"],
                                                   w.softmax_scale, out=st["pf_out"],
                                                   lse=st["pf_lse"])

    def fused(self):
        st, w = self.st, self.w
        self.pkv.paged_decode_attention_append(st["cache"], st["dec_q"], st["dec_table"],
                                               st["dec_lens"], st["dec_max"], st["k_new"],
                                               st["v_new"], w.softmax_scale, out=st["dec_out"],
                                               lse=st["dec_lse"], workspace=self.ws,
                                               num_ctas=self.num_ctas)

    def step(self):
        self.append()
        self.decode()
        self.prefill()

    def launches_per_step(self):
        # append; decode_kernel + decode_merge_kernel; prefill_kernel
        return 1 + (2 if self.has_dec else 0) + (1 if self.has_pf else 0)

    def graph(self, fn):
        """``fn``'s launches captured once into a CUDA graph (on a side stream)."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        self.gstream.wait_stream(self.stream)
        with torch.cuda.stream(self.gstream):
            fn()  # warm the caching allocator on the capture stream
            self.gstream.synchronize()
            with torch.cuda.graph(g, stream=self.gstream):
                fn()
        torch.cuda.synchronize()
        return g

    def replay_time(self, g, reps):
        """Seconds per replay of ``g``, ``reps`` replays back to back between events."""
        torch = self.torch
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(self.stream)
        for _ in range(reps):
            g.replay()
        e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / reps

    def time_alone(self, fn, min_region_s=MIN_REGION_S):
        """(seconds per call, replays) of ``fn`` graph-replayed alone, over at
        least ``min_region_s``."""
        g = self.graph(fn)
        for _ in range(3):
            g.replay()
        est = self.replay_time(g, 5)
        reps = int(min(20000, max(20, math.ceil(min_region_s / max(est, 1e-7)))))
        t = self.replay_time(g, reps)
        del g
        return t, reps

    def check_flags(self):
        f = int(self.st["flags"].item())
        if f:
            raise RuntimeError(f"device error flags {f:#x}")


def measure_workload(w, st, runner, peaks_):
    """Graph-replayed step and per-kernel times of one workload (one GPU)."""
    hbm, tf_burst, _, kind = peaks_
    step_s, step_reps = runner.time_alone(runner.step)
    dec_s = dec_reps = pf_s = pf_reps = None
    if runner.has_dec:
        dec_s, dec_reps = runner.time_alone(runner.decode)
    if runner.has_pf:
        pf_s, pf_reps = runner.time_alone(runner.prefill)
    app_s, _ = runner.time_alone(runner.append)
    runner.check_flags()
    step_bytes = decode_bytes(w) + append_bytes(w)
    e = {
        "workload": w.name,
        "kv_dtype": w.kv_dtype,
        "step_ms": round(step_s * 1e3, 5),
        "step_gbs": round(step_bytes / step_s / 1e9, 1),
        "query_tokens_per_s": round((len(w.decode_rows) + int(w.new_lens[w.chunk_rows].sum()))
                                    / step_s, 1),
        "kernels_ms": {"append": round(app_s * 1e3, 5),
                       "decode": None if dec_s is None else round(dec_s * 1e3, 5),
                       "prefill": None if pf_s is None else round(pf_s * 1e3, 5)},
        "replays": {"step": step_reps, "decode": dec_reps, "prefill": pf_reps},
        "timing": "each of the step, the decode call and the prefill call captured alone in a "
                  "CUDA graph and replayed back to back between CUDA events",
    }
    roofs = {}
    if dec_s:
        traffic = None
        prof = TRAFFIC_PROFILES.get(w.config_number)
        if prof:
            traffic = profile_traffic(prof[1], prof[2])
        roofs["decode"] = decode_roofline(dec_s, decode_bytes(w), hbm, kind, traffic)
        e["decode_gbs"] = roofs["decode"]["achieved"]
        e["decode_tokens_per_s"] = round(len(w.decode_rows) / dec_s, 1)
    if pf_s:
        roofs["prefill"] = prefill_roofline(pf_s, prefill_flops(w), tf_burst, kind)
        e["prefill_tflops"] = roofs["prefill"]["achieved"]
    e["dominant"] = "prefill" if (pf_s and (dec_s is None or pf_s > dec_s)) else "decode"
    e["roofline"] = roofs
    return e


def outputs_to_host(st):
    out = {}
    for k in ("dec_out", "dec_lse", "pf_out", "pf_lse"):
        if k in st:
            out[k] = st[k].float().cpu().numpy().astype(np.float64)
    return out


def run_ours(args, rank, world, device, dist):
    import torch
    import paged_kv_cache_476_b200 as pkv
    import workloads

    pk = peaks()
    hbm_peak, tf_burst, tf_sust, peak_kind = pk
    w = workloads.config(args.config)
    st = setup_device_state(w, device)
    r = Runner(w, st, args.num_ctas, device)
    stream = r.stream

    for _ in range(max(3, args.warmup)):
        r.step()
    torch.cuda.synchronize()
    r.check_flags()

    # Eager steps (separate launches, an event between kernels): reported as
    # "eager" beside the graph-replayed numbers.
    k_steps = max(1, min(args.steps, 300))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(k_steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(k_steps):
        e = evs[i]
        e[0].record(stream)
        r.append()
        e[1].record(stream)
        r.decode()
        e[2].record(stream)
        r.prefill()
        e[3].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    eager_s = max_over_ranks(t0.elapsed_time(t1) / 1e3 / k_steps, dist, device)
    eager_k = {"append": sum(e[0].elapsed_time(e[1]) for e in evs) / k_steps,
               "decode": sum(e[1].elapsed_time(e[2]) for e in evs) / k_steps,
               "prefill": sum(e[2].elapsed_time(e[3]) for e in evs) / k_steps}

    # Each kernel's time alone, graph-replayed like the timed steps: the
    # roofline of the dominant kernel comes from these.
    with ClockSampler(device.index if device.index is not None else 0) as kclk:
        headline = measure_workload(w, st, r, pk)
    headline["clocks"] = kclk.summary("the graph-replayed measurements of this workload")
    dec_s = headline["kernels_ms"]["decode"]
    pf_s = headline["kernels_ms"]["prefill"]

    # The timed steps: the step captured once into a CUDA graph and replayed,
    # one graph launch per step (the PDL edge between the decode kernels is
    # kept by capture).  The clock sampler runs from a soak of the same graph
    # just before the timed region through its end.
    graph = r.graph(r.step)
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()
    r.check_flags()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    soak = max(1, int(SOAK_S / max(headline["step_ms"] / 1e3, 1e-6)))
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        for _ in range(soak):
            graph.replay()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    elapsed = max_over_ranks(g0.elapsed_time(g1) / 1e3, dist, device)  # seconds
    del graph
    r.check_flags()

    # The same decode step with the append fused into the decode launch
    # (paged_decode_attention_append), graph-replayed: decode configurations
    # only, where every sequence appends one token.
    fused_s = None
    one_each = (not r.has_pf and len(w.decode_rows) == w.batch
                and bool((np.asarray(w.new_lens) == 1).all()))
    if one_each:
        fused_s, _ = r.time_alone(r.fused)
        fused_s = max_over_ranks(fused_s, dist, device)
        r.check_flags()

    # ---------------------------------------------------------------- e2e
    # Through the public API with host buffers: per step, H2D of the step's
    # inputs (q, new K/V, lengths, page table) from pinned memory and D2H of
    # the attention output, all inside the timed region.  Inputs and outputs
    # move on streams of their own with two buffers each, so step i+1's inputs
    # and step i-1's output cross PCIe while step i's kernels run.
    cache = st["cache"]
    names = ("dec_q", "k_new", "v_new", "table", "ctx_lens", "dec_lens", "dec_table")
    offs, total = {}, 0
    for k in names:
        offs[k] = total
        total += (st[k].numel() * st[k].element_size() + 255) // 256 * 256
    h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_bufs = [torch.empty(total, dtype=torch.uint8, device=device) for _ in range(2)]
    d = [{}, {}]
    for k in names:
        n = st[k].numel() * st[k].element_size()
        h_buf[offs[k]:offs[k] + n].copy_(st[k].contiguous().view(-1).view(torch.uint8).cpu())
        for i in range(2):
            d[i][k] = d_bufs[i][offs[k]:offs[k] + n].view(st[k].dtype).view(st[k].shape)
    outs = [torch.empty_like(st["dec_out"]) for _ in range(2)]
    h_outs = [torch.empty(st["dec_out"].shape, dtype=st["dec_out"].dtype).pin_memory()
              for _ in range(2)]
    h2d_stream = torch.cuda.Stream()  # inputs in
    d2h_stream = torch.cuda.Stream()  # results out
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    compute_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    e_steps = max(1, min(args.steps, 200))

    def e2e_step(i):
        b = i & 1
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(compute_done[b])  # step i-2 is done reading buffer b
            d_bufs[b].copy_(h_buf, non_blocking=True)  # one H2D copy of every step input
            h2d_done[b].record(h2d_stream)
        stream.wait_event(h2d_done[b])
        if i >= 2:
            stream.wait_event(d2h_done[b])  # step i-2's output has left outs[b]
        db = d[b]
        pkv.paged_kv_append(cache, db["table"], db["ctx_lens"], st["cu_new"], db["k_new"],
                            db["v_new"])
        pkv.paged_decode_attention(cache, db["dec_q"], db["dec_table"], db["dec_lens"],
                                   st["dec_max"], w.softmax_scale, out=outs[b], lse=st["dec_lse"],
                                   workspace=r.ws, num_ctas=args.num_ctas)
        compute_done[b].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(compute_done[b])
            h_outs[b].copy_(outs[b], non_blocking=True)  # D2H of the step's result
            d2h_done[b].record(d2h_stream)

    def e2e_run(n):
        for i in range(n):
            e2e_step(i)
        stream.wait_stream(d2h_stream)

    e2e_run(3)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d_stream.wait_event(e0)
    e2e_run(e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_s = e0.elapsed_time(e1) / 1e3 / e_steps
    e2e_s = max_over_ranks(e2e_s, dist, device)
    h2d = sum(st[k].numel() * st[k].element_size() for k in names)
    d2h = h_outs[0].numel() * h_outs[0].element_size()

    # one more plain step: its outputs are what the parity check compares
    r.step()
    torch.cuda.synchronize()
    r.check_flags()
    flags = int(st["flags"].item())
    host_out = outputs_to_host(st)
    step_bytes = decode_bytes(w) + append_bytes(w)
    step_s = elapsed / args.steps
    roof = roofline_of((dec_s or 0) / 1e3, decode_bytes(w), (pf_s or 0) / 1e3,
                       prefill_flops(w) if r.has_pf else 0, hbm_peak, tf_burst, peak_kind,
                       headline["roofline"].get("decode", {}).get("traffic"))
    res = {
        "metric": METRIC,
        "value": round(whole_job_rate(step_bytes, world, step_s) / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.kv_dtype == "bf16" else f"{w.kv_dtype}-kv/bf16-q",
        "data": "synthetic (seeded N(0,1) bf16 K/V/Q, permuted pages, NaN sentinels)",
        "tokens_per_s": round(whole_job_rate(len(w.decode_rows), world, step_s), 1),
        "config": config_dict(w, world),
        "kernels_ms": headline["kernels_ms"],
        "roofline": roof,
        "e2e": {"value": round(whole_job_rate(step_bytes, world, e2e_s) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e_s * 1e3, 5),
                "mode": "eager API calls (append + decode) per step; H2D of step i+1 and "
                        "D2H of step i-1 on their own streams, overlapping step i's kernels"},
        "timing": "value: the step (append + decode [+ prefill]) captured once in a CUDA graph "
                  "and replayed per step; kernels_ms and roofline: each call captured alone "
                  "and replayed back to back the same way",
        "eager": {"value": round(whole_job_rate(step_bytes, world, eager_s) / 1e9, 2),
                  "unit": "GB/s", "ms_per_step": round(eager_s * 1e3, 5),
                  "kernels_ms": {k: round(v, 5) for k, v in eager_k.items()},
                  "what": "the same step as separate launches, events between kernels"},
        "fused": None if fused_s is None else {
            "value": round(whole_job_rate(step_bytes, world, fused_s) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(fused_s * 1e3, 5),
            "what": "the same step with the append fused into the decode launch "
                    "(paged_decode_attention_append), graph-replayed"},
        "gpu_launches": r.launches_per_step() * args.steps,
        "clocks": clk.summary(f"a {SOAK_S:.2f} s soak of the step graph, then the timed steps"),
        "device_error_flags": flags,
    }
    if r.has_pf:
        res["prefill"] = {"tflops": headline.get("prefill_tflops"), "peak_tflops": tf_burst,
                          "flops_per_launch": int(prefill_flops(w))}
    headline["outputs"] = host_out
    del r, st
    torch.cuda.empty_cache()
    return w, res, headline


def run_per_config(configs, args, device, headline_n, headline_entry):
    """Every workload of ``configs`` measured alone on this GPU (N = 1).  Returns
    ({n: entry}, {n: (workload, host outputs)})."""
    import torch
    import workloads

    pk = peaks()
    entries, outputs = {}, {}
    for n in configs:
        if n == headline_n and headline_entry is not None:
            w = workloads.config(n)
            out = headline_entry.pop("outputs")
            entries[n] = headline_entry
            outputs[n] = (w, out)
            continue
        w = workloads.config(n)
        st = setup_device_state(w, device)
        r = Runner(w, st, args.num_ctas, device)
        for _ in range(3):
            r.step()
        torch.cuda.synchronize()
        r.check_flags()
        with ClockSampler(device.index if device.index is not None else 0) as clk:
            e = measure_workload(w, st, r, pk)
        e["clocks"] = clk.summary("the graph-replayed measurements of this workload")
        r.step()
        torch.cuda.synchronize()
        r.check_flags()
        outputs[n] = (w, outputs_to_host(st))
        entries[n] = e
        del r, st
        torch.cuda.empty_cache()
    return entries, outputs


# ----------------------------------------------------------- CPU oracle
def oracle_sample(w, n_seqs: int):
    """Decode rows for a bounded CPU sample: spread over the length range."""
    rows = w.decode_rows
    order = rows[np.argsort(w.lens_after[rows], kind="stable")]
    idx = np.linspace(0, len(order) - 1, num=min(n_seqs, len(order))).round().astype(int)
    return np.unique(order[idx])


# Bounded oracle samples per workload (decode sequences, prefill chunks):
# about 10-30 s of host work over all workloads.
ORACLE_SAMPLE = {1: (4, 0), 2: (64, 0), 3: (2, 0), 4: (64, 0), 5: (32, 2), 6: (64, 0), 7: (64, 0)}


def run_oracle(w, n_seqs: int, repeats: int = 1, one_core: bool = False):
    """Time the oracle (append of the step's tokens + decode) on a sample, on all
    host cores; with ``one_core``, also once on a single core."""
    import oracle

    sample = oracle_sample(w, n_seqs)
    c = oracle.cache_for(w, seq_ids=sample, include_new=False)
    q = oracle.bf16_bits(w.q_decode())
    k_new, v_new = w.new_kv(rows=sample)
    cu = np.concatenate([[0], np.cumsum(w.new_lens[sample])]).astype(np.int32)
    pos = {int(b): i for i, b in enumerate(w.decode_rows)}
    qi = np.array([pos[int(b)] for b in sample])
    times = []
    out = None
    for _ in range(repeats):
        t = time.perf_counter()
        c.append(w.page_table[sample], w.ctx_lens[sample], cu, oracle.bf16_bits(k_new),
                 oracle.bf16_bits(v_new))
        out = c.decode(q[qi], w.page_table[sample], w.lens_after[sample], w.softmax_scale)
        times.append(time.perf_counter() - t)
    dt = statistics.median(times)
    nbytes = decode_bytes(w, rows=sample) + append_bytes(w, rows=sample)
    single = None
    if one_core:
        # the same sample once more on one core (the append rewrites the same bytes)
        cores = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            t = time.perf_counter()
            c.append(w.page_table[sample], w.ctx_lens[sample], cu, oracle.bf16_bits(k_new),
                     oracle.bf16_bits(v_new))
            c.decode(q[qi], w.page_table[sample], w.lens_after[sample], w.softmax_scale)
            t1 = time.perf_counter() - t
        finally:
            oracle.set_num_threads(cores)
        single = {"value": round(nbytes / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                  "seconds": round(t1, 3)}
    res = {
        "value": round(nbytes / dt / 1e9, 4),
        "unit": "GB/s",
        "cores": oracle.num_threads(),
        "kind": "oracle",
        "sample": f"{len(sample)} of {len(w.decode_rows)} sequences (lengths spread over the "
                  f"range, {int(w.lens_after[sample].sum())} tokens): append + decode, fp64 C "
                  f"with OpenMP, median of {repeats}",
        "seconds": round(dt, 3),
        "tokens_per_s": round(len(sample) / dt, 3),
        "single_core": single,
    }
    return res, (qi, out)


def _bf16_round(x):
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def _parity(o, ref, lse=None, ref_lse=None):
    """max/mean |out - exact|, the worst error against the correctly rounded
    value where the first misses 1e-2, and the lse error."""
    err = np.abs(o - ref)
    res = {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
           "elements": int(err.size)}
    miss = err > 1e-2
    res["over_1e-2"] = int(miss.sum())
    if miss.any():
        res["max_abs_vs_rounded_where_over"] = float(np.abs(o - _bf16_round(ref))[miss].max())
    if lse is not None:
        fin = np.isfinite(ref_lse)
        res["lse_max_abs"] = float(np.abs(lse[fin] - ref_lse[fin]).max()) if fin.any() else 0.0
    return res


def oracle_leg(w, n, gpu_out):
    """The oracle on a bounded sample of workload ``w`` (timed, all host cores), and
    the GPU outputs of the same rows compared with it."""
    import oracle

    n_dec, n_chunks = ORACLE_SAMPLE.get(n, (16, 1))
    res = {}
    if len(w.decode_rows):
        cb, (qi, (ref, ref_lse)) = run_oracle(w, n_dec)
        res["oracle"] = cb
        # the oracle decoded the sampled rows only, in sample order
        res["parity_decode"] = _parity(gpu_out["dec_out"][qi], ref, gpu_out["dec_lse"][qi],
                                       ref_lse)
    if len(w.chunk_rows) and n_chunks:
        # the chunks with the smallest and the largest context
        order = w.chunk_rows[np.argsort(w.ctx_lens[w.chunk_rows], kind="stable")]
        pick = np.unique(order[np.linspace(0, len(order) - 1, n_chunks).round().astype(int)])
        c = oracle.cache_for(w, seq_ids=pick)
        cu_all = w.cu_q_chunks()
        qc = oracle.bf16_bits(w.q_chunks())
        pos = {int(b): i for i, b in enumerate(w.chunk_rows)}
        rows, cu = [], [0]
        for b in pick:
            i = pos[int(b)]
            rows.extend(range(cu_all[i], cu_all[i + 1]))
            cu.append(cu[-1] + cu_all[i + 1] - cu_all[i])
        rows = np.asarray(rows)
        t = time.perf_counter()
        ref, ref_lse = c.prefill_chunk(qc[rows], np.asarray(cu, np.int32), w.page_table[pick],
                                       w.lens_after[pick], w.softmax_scale)
        dt = time.perf_counter() - t
        flops = 0
        for b in pick:
            L, m = int(w.lens_after[b]), int(w.new_lens[b])
            flops += 4 * w.num_q_heads * w.head_dim * sum(L - m + i + 1 for i in range(m))
        res["oracle_prefill"] = {"seconds": round(dt, 3), "tflops": round(flops / dt / 1e12, 5),
                                 "cores": oracle.num_threads(),
                                 "sample": f"{len(pick)} of {len(w.chunk_rows)} chunks"}
        res["parity_prefill"] = _parity(gpu_out["pf_out"][rows], ref, gpu_out["pf_lse"][rows],
                                        ref_lse)
    return res


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # The reference arm is the CPU oracle; under torchrun only rank 0 works.
        if rank != 0:
            return 0
        import workloads

        w = workloads.config(args.config)
        n_seqs = args.cpu_sample_seqs
        rep = max(1, min(args.steps, 3))
        cb, _ = run_oracle(w, n_seqs, repeats=rep)
        res = {
            "metric": METRIC, "value": cb["value"], "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(cb["seconds"] * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, world),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(res))
        return 0

    import torch

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    w, res, headline = run_ours(args, rank, world, device, dist)
    if world == 1:
        configs = [int(x) for x in args.per_config.split(",") if x.strip()]
        if configs:
            entries, outs = run_per_config(configs, args, device, args.config, headline)
            if rank == 0 and not args.no_cpu_baseline:
                for n in configs:
                    wn, out = outs[n]
                    entries[n].update(oracle_leg(wn, n, out))
            res["per_config"] = {str(n): entries[n] for n in configs}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"], _ = run_oracle(w, args.cpu_sample_seqs, repeats=5, one_core=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
