#!/usr/bin/env python
"""Throughput of the HiLS attention forward pass on B200, one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hils|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...        (one process per GPU)

A step is one hils_forward call (score -> top-K -> chunk/window attention -> fusion) over one
batch of the prefill workload, inputs resident in HBM.  The default workload is the largest
single-GPU configuration: the extreme-length prefill at N = 4M tokens (B=1, 8 query heads / 1 KV
head, d=128, S=128, K=16, W=2048; 140.6 TFLOP of landmark scoring).  Steps are timed with CUDA
events recorded by the library between its kernels, so each kernel's duration comes from the
same timed steps; L2 is flushed between steps, outside the timed intervals (a 256 MiB write,
then a 256 MiB read so that the write's dirty lines reach HBM before the next step starts).
With N GPUs every rank runs its own independent batch (weak scaling, no data-path collective);
the step time is the max over ranks.

Also reported (single GPU): `e2e` (the same call from pinned host buffers, copies included),
`cpu_baseline` (the fp64 CPU oracle on a bounded sample of the same workload) with `parity`
(the GPU's outputs on the oracle-timed rows), the 4M decode step, and the other workloads of the
sweep: `prefill_small_mha` (B=4 x 16 heads x 8192 tokens), `prefill_gqa7b` (the 7B-like GQA
prefill at N=131072), `decode` (32 single-token queries over a 512K-token cache, timed as a CUDA
graph replay) and `extreme_256k` / `extreme_1m` (prefill and decode), each with per-kernel
rooflines.  `--impl reference` times the fp64 CPU oracle as the reference arm.
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import threading
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HiLS fwd prefill tokens/s & decode µs/step at 1 B200; % of HBM/TC roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in PEAKS_FALLBACK}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# --------------------------------------------------------------------------- work model
def eligible(pos, S, W):
    first = pos - W + 1
    return 0 if first <= 0 else first // S


def work_model(dims, S, K, W, q_pos0, es):
    """Algorithmic FLOPs / bytes of one forward (es = bytes per element of the inputs)."""
    B, Hq, Hkv, Nq, Nkv, d = (dims[k] for k in ("B", "Hq", "Hkv", "N_q", "N_kv", "d"))
    pos = np.arange(q_pos0, q_pos0 + Nq, dtype=np.int64)
    n = np.where(pos - W + 1 > 0, (pos - W + 1) // S, 0)
    k_sel = np.minimum(n, K)
    L = pos - S * n + 1
    C = Nkv // S
    sum_n = float(n.sum())
    tokens = float((k_sel * S + L).sum())
    m = {}
    m["score_flops"] = 2.0 * d * Hq * B * sum_n
    m["attn_flops"] = 4.0 * d * B * Hq * tokens
    # compulsory bytes of each phase (every input byte read once, every output written once)
    sel_rows, head_rows = B * Hkv * Nq, B * Hq * Nq
    if Nq <= 16:   # decode: each query reads its own landmark rows and its selected K/V
        m["select_bytes"] = B * Hkv * float((n * (d * es + 4)).sum()) + head_rows * d * es
        m["attn_bytes"] = B * Hkv * float((k_sel * S + L).sum()) * 2 * d * es + head_rows * d * es
    else:
        m["select_bytes"] = (head_rows * d * es + B * Hkv * C * (d * es + 4) +
                             sel_rows * K * 4 + head_rows * K * 4)
        m["attn_bytes"] = (head_rows * d * es * 2 + B * Hkv * Nkv * d * es * 2 +
                           sel_rows * K * 4 + head_rows * K * 4 + head_rows * 4)
    m["tokens"] = B * Nq
    return m


def phase_work(name, wm):
    """(bound, algorithmic work, unit) of a kernel, for its roofline."""
    if name in ("score_topk_tc", "score_topk_t_tc", "select_rows"):
        return "tensor", wm["score_flops"], "TFLOP/s"
    if name in ("select_split", "select_stream", "select_stream_tc"):
        return "hbm", wm["select_bytes"], "GB/s"
    if name in ("attn_units", "attn_units_tc"):
        return "hbm", wm["attn_bytes"], "GB/s"
    if name.startswith("attn"):
        return "tensor", wm["attn_flops"], "TFLOP/s"
    return "hbm", None, "GB/s"


def roofline(name, ms, wm, peaks, workload, sustained=False):
    bound, work, unit = phase_work(name, wm)
    if work is None or ms <= 0:
        return None
    if bound == "hbm":
        achieved = work / (ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
    else:
        achieved = work / (ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    return {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": traffic_for(name, workload), "work_per_launch": work}


KERNEL_SOURCES = {
    "score_topk_tc": ["score_tc.cu"], "score_topk_t_tc": ["score_t_tc.cu"],
    "attn_tc": ["attn_tc.cu"],
    "select_stream": ["select.cu"], "select_topk": ["select.cu"], "select_rows": ["select.cu"],
    "select_split": ["select.cu"], "select_stream_tc": ["stream_tc.cu"],
    "attn_units": ["attn.cu"], "attn_units_tc": ["units_tc.cu"], "attn_rows": ["attn.cu"],
    "fuse_units": ["attn.cu"], "landmarks": ["landmarks.cu"],
}
SHARED_SOURCES = ["common.cuh", "sm100.cuh"]


def code_only(text):
    """A CUDA source without its comments, whitespace runs collapsed: an edit of the comments
    leaves it unchanged, any edit of the code changes it."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return re.sub(r"\s+", " ", text).strip()


def source_sha(kernel):
    """Hash of the code of the CUDA sources a kernel is built from (its file and the shared
    headers), comments excluded."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_chunk_sparse_scoring_b200", "csrc")
    for f in KERNEL_SOURCES.get(kernel, []) + SHARED_SOURCES:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM read+write bytes per launch of `kernel` on `workload`, from the committed ncu
    summaries (profiles/traffic.json), if they were taken on the kernel's current source;
    else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get("%s@%s" % (kernel, workload))
        if not rec or kernel not in KERNEL_SOURCES:
            return None
        return rec["bytes_per_launch"] if rec.get("source_sha") == source_sha(kernel) else None
    except Exception:
        return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML from a thread while the
    timed region runs (read-only queries; no setting is touched)."""
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("sw_power_cap", 0x4))

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.rows = []
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()
        self._thread = None

    def _handle(self, nv):
        try:
            pr = torch.cuda.get_device_properties(self.cuda_index)
            bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _poll(self, nv, h):
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while True:
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = reasons_fn(h)
                self.rows.append((float(mhz), int(bits)))
            except Exception as e:       # keep whatever was sampled
                self.err = repr(e)
                return
            if self._stop.wait(0.001):
                return

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self._thread.start()
        except Exception as e:
            self.err = repr(e)
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.rows:
            return None
        reasons = sorted({name for _, bits in self.rows for name, m in self.REASONS if bits & m})
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.rows), "source": "nvml"}


# --------------------------------------------------------------------------- timing
def make_events(n):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()          # materialise the CUDA event handles
    torch.cuda.synchronize()
    return evs


class Runner:
    """Preallocated buffers for repeated hils_forward calls on one workload."""

    def __init__(self, wl):
        from hierarchical_chunk_sparse_scoring_b200 import binding as hb
        self.hb = hb
        self.wl = wl
        self.p = hb.params_for(wl.q, wl.K, **wl.kwargs())
        self.phases = hb.phases(self.p)
        B, Hq, Nq, d = wl.q.shape
        self.out = torch.empty_like(wl.q)
        self.lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=wl.q.device)
        self.idx = torch.empty((B, wl.K.shape[1], Nq, wl.K_top), dtype=torch.int32,
                               device=wl.q.device)
        self.ws = hb.workspace(self.p, wl.q.device)

    def __call__(self, events=None, inputs=None):
        wl = self.wl
        q, qc, K, V, klm, blm = inputs or (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)
        self.hb.forward_raw(self.p, q, qc, K, V, klm, blm, self.out, self.lse, self.idx, self.ws,
                            events=events)


def timed_steps(run, steps, flush, barrier=lambda: None):
    n_ph = len(run.phases)
    evs = [make_events(n_ph + 1) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for k in range(steps):
        flush()
        run(events=evs[k])
    torch.cuda.synchronize()
    barrier()
    step_ms = [evs[k][0].elapsed_time(evs[k][-1]) for k in range(steps)]
    phase_ms = {name: statistics.mean(evs[k][j].elapsed_time(evs[k][j + 1]) for k in range(steps))
                for j, name in enumerate(run.phases)}
    return step_ms, phase_ms


def make_flush(device):
    """Evicts the previous step's data from L2: a write of a buffer larger than L2, then a read
    of another one, whose clean lines displace the write's dirty ones (otherwise their write-back
    to HBM would fall inside the next timed step)."""
    buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    src = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    acc = torch.empty((), dtype=torch.float32, device=device)

    def flush():
        buf.fill_(1.0)
        torch.sum(src, dim=0, out=acc)
    return flush


# --------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, seconds, rng_seed=0, max_rows=None, cache=None):
    """Times the fp64 oracle on randomly chosen (b, g, query) rows of `wl` (all G heads of each
    row), sized to run about `seconds`.  Returns a dict: tokens/s, rows, threads, wall seconds,
    and the rows with the oracle's results (for the parity summary)."""
    import oracle
    Hq, d = wl.q.shape[1], wl.q.shape[3]
    Hkv = wl.K.shape[1]
    G = Hq // Hkv
    B, Nq = wl.q.shape[0], wl.q.shape[2]
    rng = np.random.default_rng(rng_seed)
    cache = {} if cache is None else cache

    def f64(t):
        # converted on the tensor's own device, then copied to the host once
        return t.detach().to(torch.float64).cpu().numpy()

    def build(n_rows):
        picks, qs = [], []
        for _ in range(n_rows):
            b, g, i = int(rng.integers(B)), int(rng.integers(Hkv)), int(rng.integers(Nq))
            if (b, g) not in cache:
                cache[(b, g)] = (f64(wl.k_lm[b, g]), f64(wl.b_lm[b, g]), f64(wl.K[b, g]),
                                 f64(wl.V[b, g]))
            klm, blm, kr, vr = cache[(b, g)]
            picks.append((b, g, i))
            qs.append(oracle.Query(wl.q_pos0 + i, f64(wl.q[b, g * G:(g + 1) * G, i]),
                                   f64(wl.q_cal[b, g * G:(g + 1) * G, i]), klm, blm, kr, vr))
        return picks, qs

    threads = oracle.default_threads()
    kw = dict(d=d, G=G, S=wl.S, K_top=wl.K_top, W=wl.W, threads=threads)
    rows = max(threads, 8)
    while True:
        picks, qs = build(rows)
        t0 = time.perf_counter()
        res = oracle.run_queries(qs, **kw)
        dt = time.perf_counter() - t0
        if dt >= seconds * 0.5 or (max_rows and rows >= max_rows):
            break
        rows = int(min(rows * max(2.0, seconds / max(dt, 1e-3)), max_rows or 1 << 30))
    tokens = rows * G / Hq
    return {"rate": tokens / dt, "rows": rows, "threads": threads, "seconds": dt,
            "picks": picks, "results": res}


def oracle_sample_rate(wl, seconds, rng_seed=0, max_rows=None, cache=None):
    r = oracle_sample(wl, seconds, rng_seed, max_rows, cache)
    return r["rate"], r["rows"], r["threads"], r["seconds"]


def parity_summary(run, sample, gap_tol=1e-3):
    """The GPU run's outputs on the oracle-timed rows: how many rows select exactly the oracle's
    chunks (rows whose rank-K gap exceeds gap_tol), how many are near ties, and the largest
    output / log-sum-exp differences on the rows whose selection matches."""
    wl = run.wl
    G = wl.q.shape[1] // wl.K.shape[1]
    K = wl.K_top
    clear = match = ties = 0
    out_err = lse_err = 0.0
    for (b, g, i), r in zip(sample["picks"], sample["results"]):
        gsel = run.idx[b, g, i].cpu().numpy()
        osel = r["idx"]
        same_set = set(int(c) for c in gsel if c >= 0) == set(int(c) for c in osel if c >= 0)
        if r["gap"] > gap_tol:
            clear += 1
            match += int(same_set)
        else:
            ties += 1
        if same_set:
            o = run.out[b, g * G:(g + 1) * G, i].double().cpu().numpy()
            l = run.lse[b, g * G:(g + 1) * G, i].double().cpu().numpy()
            out_err = max(out_err, float(np.abs(o - r["out"]).max()))
            lse_err = max(lse_err, float(np.abs(l - r["lse"]).max()))
    return {"rows": len(sample["picks"]), "clear_gap_rows": clear,
            "idx_match_rate": (match / clear) if clear else None, "near_tie_rows": ties,
            "out_abs_max": out_err, "lse_abs_max": lse_err, "K": K,
            "rule": "sets equal where the oracle's rank-K gap > 1e-3; errors on matching rows"}


# --------------------------------------------------------------------------- arms
HEADLINE = ("extreme", 1 << 22)   # the extreme-length prefill at N = 4M tokens


def workload_N(args):
    if args.N is None and args.workload == HEADLINE[0]:
        return HEADLINE[1]
    return args.N


def primary_workload(args, device, rank):
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    seed = W.SPECS[args.workload]["seed"] + 1000 * rank
    return W.make(args.workload, device, seed=seed, N=workload_N(args), B=args.B)


def config_of(wl, n_gpus):
    d = wl.dims
    return {"workload": wl.name, "B": d["B"], "Hq": d["Hq"], "Hkv": d["Hkv"], "N": d["N_kv"],
            "d": d["d"], "S": wl.S, "K_top": wl.K_top, "W": wl.W,
            "global_batch": d["B"] * n_gpus, "seq_len": d["N_kv"],
            "parallelism": "dp%d (independent batches per GPU)" % n_gpus,
            "l2": "flushed between steps (256 MiB write, then 256 MiB read), outside the "
                  "timed intervals"}


def measure_e2e(run, steps, warmup):
    """The same call from pinned host buffers: every step copies all of its inputs host to device,
    runs the forward and copies its output back.  Steps are pipelined over two buffer sets: the
    copies of one step overlap the forward of the previous one (host-to-device and device-to-host
    on separate streams), as a serving loop would run them.  The serial form (one step at a time)
    is reported beside it."""
    wl = run.wl
    host = [t.cpu().pin_memory() for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    runs = [run, Runner(wl)]
    # the second buffer set's forward gets a workspace of its own (two forwards in flight)
    runs[1].ws = runs[1].hb.workspace(runs[1].p, wl.q.device, stream=s_comp)
    devs = [[torch.empty_like(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
            for _ in range(2)]
    outs = [torch.empty(run.out.shape, dtype=run.out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = outs[0].numel() * outs[0].element_size()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_done + ev_out:
        e.record(s_comp)

    def step(k):
        sl = k & 1
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[sl])          # the forward of step k-2 has read this set
            for d_, h_ in zip(devs[sl], host):
                d_.copy_(h_, non_blocking=True)
            ev_in[sl].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[sl])
            s_comp.wait_event(ev_out[sl])         # step k-2's output has been copied out
            runs[sl](inputs=devs[sl])
            ev_done[sl].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[sl])
            outs[sl].copy_(runs[sl].out, non_blocking=True)
            ev_out[sl].record(s_out)

    def timed(n, pipelined):
        torch.cuda.synchronize()
        a, b = make_events(2)
        a.record(s_in)
        for k in range(n):
            step(k)
            if not pipelined:
                s_in.wait_stream(s_out)
        s_in.wait_stream(s_out)
        b.record(s_in)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    for k in range(warmup):
        step(k)
    t = timed(steps, True)
    t_serial = timed(steps, False)
    return {"value": wl.q.shape[0] * wl.q.shape[2] / (t * 1e-3), "unit": "tokens/s",
            "ms_per_step": t, "ms_per_step_serial": t_serial,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "two buffer sets; copies of a step overlap the previous forward"}


def extra_prefill(name, steps, peaks, **overrides):
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    wl = W.make(name, "cuda", **overrides)
    run = Runner(wl)
    flush = make_flush(wl.q.device)
    run()
    torch.cuda.synchronize()
    step_ms, phase_ms = timed_steps(run, steps, flush)
    es = wl.q.element_size()
    wm = work_model(wl.dims, wl.S, wl.K_top, wl.W, wl.q_pos0, es)
    t = statistics.mean(step_ms)
    G = wl.q.shape[1] // wl.K.shape[1]
    res = {"workload": name, "ms_per_step": t, "tokens_per_s": wm["tokens"] / (t * 1e-3),
           "union_per_K_128_rows": union_stat(run.idx, 128 // G, wl.K.shape[2] // wl.S),
           "phases_ms": phase_ms,
           "rooflines": [roofline(k, v, wm, peaks, name) for k, v in phase_ms.items()],
           "score_tflop": wm["score_flops"] / 1e12, "attn_tflop": wm["attn_flops"] / 1e12}
    del run, wl
    torch.cuda.empty_cache()
    return res


def graph_step_ms(run, steps, flush):
    """Device time of one forward as a CUDA graph replay (how the pages time decode, [Reader]
    Fig. 6), median over `steps` replays with L2 flushed before each."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        run()
    g.replay()
    torch.cuda.synchronize()
    gms = []
    for _ in range(steps):
        flush()
        a, b = make_events(2)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        gms.append(a.elapsed_time(b))
    del g
    return statistics.median(gms)


def extra_decode(steps, peaks, **overrides):
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    wl = W.make("long_decode", "cuda", **overrides)
    run = Runner(wl)
    flush = make_flush(wl.q.device)
    run()
    torch.cuda.synchronize()
    step_ms, phase_ms = timed_steps(run, steps, flush)
    # the step as one CUDA graph replay (the pages time decode with CUDA graphs)
    gms = [graph_step_ms(run, steps, flush)]
    es = wl.q.element_size()
    wm = work_model(wl.dims, wl.S, wl.K_top, wl.W, wl.q_pos0, es)
    total_bytes = wm["select_bytes"] + wm["attn_bytes"]
    t_us = statistics.median(gms) * 1e3
    res = {"workload": "long_decode", "us_per_step": t_us,
           "us_per_step_eager": statistics.mean(step_ms) * 1e3, "phases_ms": phase_ms,
           "step_bytes": total_bytes,
           "step_roofline": {"bound": "hbm", "achieved": total_bytes / (t_us * 1e-6) / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": total_bytes / (t_us * 1e-6) / 1e9 / peaks["hbm_gbs"]},
           "rooflines": [roofline(k, v, wm, peaks, "long_decode") for k, v in phase_ms.items()]}
    del run, wl
    torch.cuda.empty_cache()
    return res


def extra_decode_step(steps, peaks):
    """hils_decode_step on the long-decode cache (32 sequences, 512K tokens, 32/8 heads): append
    the token, build the landmark of the chunk it completes, and the forward for its query, as one
    CUDA graph replay; at a chunk boundary (pos = N - 1) and inside a chunk (pos = N - 2)."""
    from hierarchical_chunk_sparse_scoring_b200 import binding as hb
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    wl = W.make("long_decode", "cuda")
    B, Hq, _, d = wl.q.shape
    Hkv, N = wl.K.shape[1], wl.K.shape[2]
    g = torch.Generator(device="cuda").manual_seed(99)
    k_new = wl.K[:, :, -1].clone()
    v_new = wl.V[:, :, -1].clone()
    q_lm = (torch.randn((B, Hkv, d), generator=g, device="cuda") / math.sqrt(d)).to(wl.q.dtype)
    flush = make_flush(wl.q.device)
    res = {"workload": "long_decode", "B": B, "N": N}
    for label, pos in (("chunk_boundary", N - 1), ("inside_chunk", N - 2)):
        p = hb.make_params(B, Hq, Hkv, 1, N, d, S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=pos)
        s = torch.cuda.Stream()
        out = torch.empty_like(wl.q)
        lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
        idx = torch.empty((B, Hkv, 1, wl.K_top), dtype=torch.int32, device="cuda")
        ws = hb.workspace(p, wl.q.device, stream=s)

        def call():
            hb.decode_step(wl.q, wl.q_cal, k_new, v_new, q_lm, wl.K, wl.V, wl.k_lm, wl.b_lm,
                           pos=pos, S=wl.S, K_top=wl.K_top, W=wl.W, out=out, lse=lse, idx=idx,
                           ws=ws, stream=s)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            call()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            call()
        graph.replay()
        torch.cuda.synchronize()
        us = []
        for _ in range(steps):
            flush()
            a, b_ = make_events(2)
            a.record()
            graph.replay()
            b_.record()
            torch.cuda.synchronize()
            us.append(a.elapsed_time(b_) * 1e3)
        del graph
        wm = work_model(dict(B=B, Hq=Hq, Hkv=Hkv, N_q=1, N_kv=N, d=d), wl.S, wl.K_top, wl.W, pos,
                        wl.q.element_size())
        nbytes = wm["select_bytes"] + wm["attn_bytes"] + 2 * B * Hkv * d * 2 * 2
        if pos == N - 1:
            nbytes += B * Hkv * (wl.S * d * 2 + 2 * d * 2 + 4)
        t = statistics.median(us)
        res[label] = {"pos": pos, "us_per_step": t, "step_bytes": nbytes,
                      "hbm_frac": nbytes / (t * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    del wl
    torch.cuda.empty_cache()
    return res


def union_stat(idx, tq, C):
    """Mean number of distinct chunks selected by tq adjacent queries of a KV group, divided by
    K (how much the packed attention shares chunk loads)."""
    R, Nq, K = idx.shape[0] * idx.shape[1], idx.shape[2], idx.shape[3]
    nt = Nq // tq
    if nt == 0 or K == 0:
        return None
    x = idx.reshape(R, Nq, K)[:, :nt * tq].reshape(R * nt, tq * K).long()
    valid = (x >= 0) & (x < C)
    hit = torch.zeros((R * nt, C + 1), dtype=torch.bool, device=idx.device)
    hit.scatter_(1, torch.where(valid, x, torch.full_like(x, C)), True)
    sizes = hit[:, :C].sum(1).float()
    return float(sizes.mean().item()) / K


def time_mode(wl, steps, peaks, label):
    """Timed hils_forward steps of one workload (prefill or decode) with per-kernel rooflines."""
    run = Runner(wl)
    flush = make_flush(wl.q.device)
    run()
    torch.cuda.synchronize()
    step_ms, phase_ms = timed_steps(run, steps, flush)
    wm = work_model(wl.dims, wl.S, wl.K_top, wl.W, wl.q_pos0, wl.q.element_size())
    t = statistics.mean(step_ms)
    res = {"ms_per_step": t, "phases_ms": phase_ms,
           "rooflines": [roofline(k, v, wm, peaks, label) for k, v in phase_ms.items()]}
    if wl.q.shape[2] > 16:
        res["tokens_per_s"] = wm["tokens"] / (t * 1e-3)
        res["score_tflop"] = wm["score_flops"] / 1e12
        res["attn_tflop"] = wm["attn_flops"] / 1e12
    else:
        # decode: the step as one CUDA graph replay; the phase split comes from the eager steps
        # (events recorded between the kernels)
        tg = graph_step_ms(run, steps, flush)
        res["us_per_step"] = tg * 1e3
        res["us_per_step_eager"] = t * 1e3
        res["step_bytes"] = wm["select_bytes"] + wm["attn_bytes"]
        res["step_hbm_frac"] = res["step_bytes"] / (tg * 1e-3) / 1e9 / peaks["hbm_gbs"]
    del run
    return res


def extra_extreme(steps, peaks, N=262144):
    """One point of the extreme-length sweep: prefill of the whole sequence and one decode
    step of its last query, on the same inputs."""
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    wl = W.make("extreme", "cuda", N=N)
    res = {"workload": "extreme", "N": N,
           "prefill": time_mode(wl, steps, peaks, "extreme_N%d" % N),
           "decode": time_mode(W.decode_view(wl), max(steps, 5), peaks, "extreme_N%d_decode" % N)}
    del wl
    torch.cuda.empty_cache()
    return res


def extra_landmarks(peaks, B, Hkv, N, d, S, steps=5, seed=77):
    """Landmark construction (hils_landmarks) over a whole cache: every key read once, one
    summary row and bias written per chunk; HBM-bound."""
    from hierarchical_chunk_sparse_scoring_b200 import binding as hb
    g = torch.Generator(device="cuda").manual_seed(seed)
    C = N // S
    K = (torch.randn((B, Hkv, N, d), generator=g, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    q_lm = (torch.randn((B, Hkv, C, d), generator=g, device="cuda") /
            math.sqrt(d)).to(torch.bfloat16)
    k_lm = torch.empty((B, Hkv, C, d), dtype=torch.bfloat16, device="cuda")
    b_lm = torch.empty((B, Hkv, C), dtype=torch.float32, device="cuda")
    flush = make_flush(K.device)
    hb.landmarks(q_lm, K, S=S, k_lm=k_lm, b_lm=b_lm)
    ms = []
    for _ in range(steps):
        flush()
        a, b_ = make_events(2)
        a.record()
        hb.landmarks(q_lm, K, S=S, k_lm=k_lm, b_lm=b_lm)
        b_.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b_))
    t = statistics.mean(ms)
    nbytes = B * Hkv * (N * d * 2 + C * d * 2 * 2 + C * 4)
    gbs = nbytes / (t * 1e-3) / 1e9
    del K, q_lm, k_lm, b_lm
    torch.cuda.empty_cache()
    return {"kernel": "landmarks", "shape": {"B": B, "Hkv": Hkv, "N": N, "d": d, "S": S},
            "ms": t, "bytes": nbytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"]}}


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz (the
# backward's products run there; no measured figure exists for this unit)
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def extra_backward(peaks, name="gqa7b_prefill", steps=3, **overrides):
    """hils_backward on a prefill workload, the forward's own selection held fixed.  Algorithmic
    FLOPs: 10 d per (row, attended token) (the logits and dout . V recomputed, then the dq, dK
    and dV products) plus 4 d per (row, selected slot) (d q_cal and d k_lm)."""
    from hierarchical_chunk_sparse_scoring_b200 import binding as hb
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    wl = W.make(name, "cuda", **overrides)
    kw = wl.kwargs()
    _, _, idx = hb.forward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, **kw)
    g = torch.Generator(device="cuda").manual_seed(5)
    dout = torch.randn(wl.q.shape, generator=g, device="cuda").to(wl.q.dtype)
    dlse = torch.randn(wl.q.shape[:3], generator=g, device="cuda")
    p = hb.make_params(*[wl.dims[k] for k in ("B", "Hq", "Hkv", "N_q", "N_kv", "d")], S=wl.S,
                       K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0, dtype=wl.q.dtype)
    ws = hb.backward_workspace(p, wl.q.device)
    grads = hb.backward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, idx, dout, dlse, ws=ws,
                        **kw)
    flush = make_flush(wl.q.device)
    ms = []
    for _ in range(steps):
        flush()
        a, b_ = make_events(2)
        a.record()
        hb.backward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, idx, dout, dlse, ws=ws,
                    out=grads, **kw)
        b_.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b_))
    t = statistics.mean(ms)
    wm = work_model(wl.dims, wl.S, wl.K_top, wl.W, wl.q_pos0, wl.q.element_size())
    pos = np.arange(wl.q_pos0, wl.q_pos0 + wl.dims["N_q"], dtype=np.int64)
    n = np.where(pos - wl.W + 1 > 0, (pos - wl.W + 1) // wl.S, 0)
    slots = float(np.minimum(n, wl.K_top).sum()) * wl.dims["B"] * wl.dims["Hq"]
    flops = 2.5 * wm["attn_flops"] + 4.0 * wl.dims["d"] * slots
    tf = flops / (t * 1e-3) / 1e12
    if wl.q.dtype == torch.bfloat16:   # products on the tensor cores (m16n8k16 bf16 tiles)
        rl = {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
              "frac": tf / peaks["bf16_tflops"]}
    else:                              # fp32 products on the CUDA cores
        rl = {"bound": "alu", "achieved": tf, "peak": FP32_FMA_TFLOPS, "unit": "TFLOP/s",
              "frac": tf / FP32_FMA_TFLOPS,
              "peak_note": "fp32 FMA of the CUDA cores, 148 SMs x 128 lanes x 2 x 1.965 GHz"}
    out = {"kernel": "bwd_rows + bwd_keys (+ index build)", "workload": name,
           "shape": {k: wl.dims[k] for k in ("B", "Hq", "Hkv", "N_q", "N_kv", "d")},
           "ms": t, "tflop": flops / 1e12, "tokens_per_s": wl.dims["B"] * wl.dims["N_q"] / (t * 1e-3),
           "roofline": rl}
    del wl, grads, ws, dout, dlse, idx
    torch.cuda.empty_cache()
    return out


def extra_prologue(peaks, B=1, Hq=32, N=131072, d=128, d_model=4096, r=16, steps=5):
    """hils_qcal_hope at the 7B-like prefill shape: the down-projection GEMM
    ([B N, d_model] x [Hq r, d_model]^T, tcgen05) and the fused up-projection + HoPE pass
    (q read, u read, q and q_cal written)."""
    from hierarchical_chunk_sparse_scoring_b200 import binding as hb
    g = torch.Generator(device="cuda").manual_seed(21)
    bf = torch.bfloat16
    q = (torch.randn((B, Hq, N, d), generator=g, device="cuda") / math.sqrt(d)).to(bf)
    hidden = torch.randn((B, N, d_model), generator=g, device="cuda").to(bf)
    W_down = (torch.randn((Hq, r, d_model), generator=g, device="cuda") /
              math.sqrt(d_model)).to(bf)
    W_up = (0.1 * torch.randn((Hq, d, r), generator=g, device="cuda")).to(bf)
    q_out, q_cal = torch.empty_like(q), torch.empty_like(q)
    kw = dict(rope_base=10000.0, train_len=32768.0, q_out=q_out, q_cal_out=q_cal)
    hb.qcal_hope(q, hidden, W_down, W_up, **kw)
    flush = make_flush(q.device)
    ms = []
    for _ in range(steps):
        flush()
        a, b_ = make_events(2)
        a.record()
        hb.qcal_hope(q, hidden, W_down, W_up, **kw)
        b_.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b_))
    t = statistics.mean(ms)
    gemm_flops = 2.0 * B * N * Hq * r * d_model
    gemm_bytes = B * N * d_model * 2 + Hq * r * d_model * 2 + B * N * Hq * r * 4
    pass_bytes = B * Hq * N * d * 2 * 3 + B * N * Hq * r * 4
    # lower bound of the pair: the GEMM at the bf16 peak plus the pass at the HBM peak
    floor_ms = (gemm_flops / (peaks["bf16_tflops"] * 1e12) +
                (gemm_bytes + pass_bytes) / (peaks["hbm_gbs"] * 1e9)) * 1e3
    del q, hidden, W_down, W_up, q_out, q_cal
    torch.cuda.empty_cache()
    return {"kernel": "qdown (tcgen05) + qcal_hope", "shape": {"B": B, "Hq": Hq, "N": N, "d": d,
            "d_model": d_model, "r": r}, "ms": t, "gemm_tflop": gemm_flops / 1e12,
            "bytes": gemm_bytes + pass_bytes, "floor_ms": floor_ms, "frac_of_floor": floor_ms / t}


def run_hils(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the HiLS path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    barrier = (lambda: dist.barrier()) if dist else (lambda: None)
    peaks, peaks_src = load_peaks()

    wl = primary_workload(args, device, rank)
    run = Runner(wl)
    flush = make_flush(device)
    for _ in range(args.warmup):
        flush()
        run()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        step_ms, phase_ms = timed_steps(run, args.steps, flush, barrier)
    from hierarchical_chunk_sparse_scoring_b200 import sharding
    total_ms = sharding.max_over_ranks(sum(step_ms), device=device if dist else None)
    ms_per_step = total_ms / args.steps
    tokens_per_rank = wl.q.shape[0] * wl.q.shape[2]
    value = sharding.aggregate_tokens_per_s(tokens_per_rank, ms_per_step, world)
    es = wl.q.element_size()
    wm = work_model(wl.dims, wl.S, wl.K_top, wl.W, wl.q_pos0, es)
    dom = max(phase_ms, key=phase_ms.get)
    label = wl.name if workload_N(args) is None else "%s_N%d" % (wl.name, wl.dims["N_kv"])
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.q.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded generator, hierarchical_chunk_sparse_scoring_b200/workloads.py)",
        "config": config_of(wl, world),
        "roofline": roofline(dom, phase_ms[dom], wm, peaks, label),
        "rooflines": [roofline(k, v, wm, peaks, label) for k, v in phase_ms.items()],
        "peaks_source": peaks_src,
        "phases_ms": phase_ms,
        "score_tflop": wm["score_flops"] / 1e12, "attn_tflop": wm["attn_flops"] / 1e12,
        "gpu_launches": len(run.phases) * args.steps,
        "union_per_K_128_rows": union_stat(run.idx, 128 // (wl.q.shape[1] // wl.K.shape[1]),
                                           wl.K.shape[2] // wl.S),
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_extras:
        line["e2e"] = measure_e2e(run, max(3, args.steps // 4), 1)
        torch.cuda.empty_cache()
        sample = oracle_sample(wl, args.cpu_seconds)
        line["cpu_baseline"] = {"value": sample["rate"], "unit": "tokens/s",
                                "cores": sample["threads"], "kind": "oracle",
                                "sample": "%d random (b, kv-group, query) rows of %s, all heads "
                                          "of each group, %.1f s wall" % (
                                              sample["rows"], label, sample["seconds"])}
        line["parity"] = parity_summary(run, sample)
        del sample, run
        torch.cuda.empty_cache()
        if wl.name == "extreme":
            from hierarchical_chunk_sparse_scoring_b200 import workloads as W
            line["extreme_%dk_decode" % (wl.dims["N_kv"] >> 10)] = time_mode(
                W.decode_view(wl), max(5, args.steps), peaks, label + "_decode")
        del wl
        torch.cuda.empty_cache()
        line["prefill_small_mha"] = extra_prefill("small_mha_bf16", 5, peaks)
        line["prefill_gqa7b"] = extra_prefill("gqa7b_prefill", 3, peaks)
        line["decode"] = extra_decode(max(5, args.steps), peaks)
        line["decode_step"] = extra_decode_step(max(5, args.steps), peaks)
        line["extreme_256k"] = extra_extreme(3, peaks, N=1 << 18)
        line["extreme_1m"] = extra_extreme(2, peaks, N=1 << 20)
        line["landmarks"] = [extra_landmarks(peaks, 1, 1, 1 << 22, 128, 128),
                             extra_landmarks(peaks, 1, 8, 131072, 128, 64)]
        line["backward_gqa7b"] = extra_backward(peaks, "gqa7b_prefill")
        line["prologue_gqa7b"] = extra_prologue(peaks)
    if dist:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on the host cores."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from hierarchical_chunk_sparse_scoring_b200 import workloads as W
    # the same seeded inputs as the GPU arm (drawn on the GPU when there is one: the generator
    # streams differ between devices); the oracle itself runs on the host cores
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = W.make(args.workload, dev, N=workload_N(args), B=args.B)
    per_step = max(1.0, args.ref_step_seconds)
    rates, rows_total, threads = [], 0, 1
    cache = {}   # the (b, g) landmark and K/V arrays in fp64, converted once
    for k in range(args.warmup + args.steps):
        rate, rows, threads, dt = oracle_sample_rate(wl, per_step if k >= args.warmup else 1.0,
                                                     rng_seed=k, cache=cache)
        if k >= args.warmup:
            rates.append(rate)
            rows_total += rows
    value = statistics.mean(rates)
    n_tokens = wl.q.shape[0] * wl.q.shape[2]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": n_tokens / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generator, hierarchical_chunk_sparse_scoring_b200/workloads.py)",
            "config": config_of(wl, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle",
                             "sample": "%d random (b, kv-group, query) rows over %d steps, "
                                       "extrapolated to the full batch" % (rows_total, args.steps)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_only_extra(args):
    """One extra measurement on its own (the commands the profiles/ summaries were taken with)."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the HiLS path has no CPU fallback)")
    peaks, _ = load_peaks()
    n = args.N
    if args.only_extra == "backward":
        out = extra_backward(peaks, args.workload if args.workload != HEADLINE[0] else
                             "gqa7b_prefill", steps=args.steps, **({"N": n} if n else {}))
    elif args.only_extra == "prologue":
        out = extra_prologue(peaks, N=n or 131072, steps=args.steps)
    elif args.only_extra == "decode":
        out = extra_decode(max(3, args.steps), peaks)
    elif args.only_extra == "decode_step":
        out = extra_decode_step(max(3, args.steps), peaks)
    elif args.only_extra == "extreme_decode":
        from hierarchical_chunk_sparse_scoring_b200 import workloads as W
        N = n or 262144
        wl = W.make("extreme", "cuda", N=N)
        out = {"workload": "extreme", "N": N,
               "decode": time_mode(W.decode_view(wl), max(5, args.steps), peaks,
                                   "extreme_N%d_decode" % N)}
    else:
        out = extra_landmarks(peaks, 1, 1, n or (1 << 22), 128, 128, steps=args.steps)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["hils", "reference"], default="hils")
    ap.add_argument("--workload", default=HEADLINE[0])
    ap.add_argument("--N", type=int, default=None, help="override the workload's sequence length")
    ap.add_argument("--B", type=int, default=None, help="override the workload's batch")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--only-extra", choices=["backward", "prologue", "decode", "decode_step",
                                             "extreme_decode", "landmarks"], default=None,
                    help="run one extra measurement alone and print its JSON (for profiling)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "hils":
        args.warmup = 3
    if args.only_extra:
        run_only_extra(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_hils(args)


if __name__ == "__main__":
    main()
