#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet layer on B200: one JSON line on stdout (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline: one gdn_chunk_prefill of the long-context workload (one sequence of T = 262,144
tokens, the model card's native context; 16 key heads, 32 value heads, d = 128, bf16
activations, fp32 state; conv + SiLU + L2 norms + gated delta rule + gated RMSNorm, final
recurrent and conv states returned), inputs resident in HBM, L2 flushed between timed steps.
Each timed step is one replay of the step's CUDA graph, with the library's launch trace
captured into the graph, so the per-kernel times (and the dominant kernel's roofline) come
from the same timed replays.  `value` is whole-job tokens/s.  Alongside: the T = 4096 and the
8-sequence variable-length prefill workloads (same figures each), an end-to-end figure of the
headline through the C ABI with host buffers, the decode workload (256 sequences x 64 steps,
state GB/s) and its bf16-state and 4-token variants, and the fp64 CPU oracle timed on this
host on a bounded sample.  N > 1 (torchrun, one process per GPU) runs independent replicas
(the layer needs no collective): weak scaling, max time over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gated_deltanet_layer_02_b200 import inputs  # noqa: E402

METRIC = "prefill tokens/s per GDN layer (% TC peak); decode state GB/s (% HBM peak)"
CHUNK = 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------- work per token
def flops_per_token_by_kernel(w, C=CHUNK):
    """Useful (triangle-masked) chunk-form FLOPs per token, split by the kernel that does them.
    Their sum is F(C) = 2 [Hv (3 d^2 + 1.5 C d + C^2/6) + Hk C d].  The q/k/v kernel (conv,
    SiLU, norms) does no contraction."""
    Hv, Hk, d = w.num_v_heads, w.num_k_heads, w.head_dim
    f = {
        "gdn_qkv": 0.0,
        "gdn_prep": 2.0 * (Hv * (C * d + C * C / 6.0) + Hk * C * d / 2.0),   # K K^T, solve, W, U~
        "gdn_chain": 2.0 * (Hv * 2.0 * d * d),                               # W S^T, K^T U
        "gdn_out": 2.0 * (Hv * (d * d + C * d / 2.0) + Hk * C * d / 2.0),    # Q K^T, Q S^T, P U
    }
    return f


def bytes_per_token_by_kernel(w):
    """Algorithmic HBM bytes per token (the layer's own inputs and outputs), by the kernel that
    moves them: x in gdn_qkv; beta, g in gdn_prep; z in and the output in gdn_out."""
    esz = 2 if w.dtype == torch.bfloat16 else 4
    Hv, d = w.num_v_heads, w.head_dim
    b = {"gdn_qkv": w.channels * esz, "gdn_prep": 2 * Hv * 4, "gdn_chain": 0,
         "gdn_out": 2 * Hv * d * esz}
    return b


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            m = json.load(f)
        return {k: float(m[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# source files of each kernel family (a change to any of them invalidates its ncu traffic figure)
KERNEL_SOURCES = {
    "prefill": ("prefill_tc.cu", "args.cuh", "common.cuh", "tc.cuh"),
    "decode_step": ("decode.cu", "args.cuh", "common.cuh", "tc.cuh"),
}


def source_hash(family="prefill"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_deltanet_layer_02_b200", "csrc")
    for name in KERNEL_SOURCES[family]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, tokens_per_launch=None):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's sources are unchanged.
    A prefill capture covers `capture_tokens` tokens per launch; the figure is scaled to
    `tokens_per_launch` (the traffic of these kernels grows with the chunks they process)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
    except Exception:
        return None
    k = t.get("kernels", {}).get(kernel)
    family = "decode_step" if kernel.startswith("decode") else "prefill"
    if k is None or k.get("source_hash") != source_hash(family):
        return None
    b = float(k["dram_bytes_per_launch"])
    if tokens_per_launch is not None and k.get("capture_tokens"):
        b *= tokens_per_launch / float(k["capture_tokens"])
    return b


# ------------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls NVML for SM clock and throttle reasons while the timed region runs."""

    HW_SLOWDOWN = 0x8
    SW_THERMAL = 0x20
    HW_THERMAL = 0x40
    SW_POWER_CAP = 0x4

    def __init__(self, index):
        self.index, self.samples, self.reasons = index, [], 0
        self._stop = threading.Event()
        self._t = None
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        names = []
        if self.reasons & self.HW_SLOWDOWN:
            names.append("hw_slowdown")
        if self.reasons & self.HW_THERMAL:
            names.append("hw_thermal_slowdown")
        if self.reasons & self.SW_THERMAL:
            names.append("sw_thermal_slowdown")
        if self.reasons & self.SW_POWER_CAP:
            names.append("sw_power_cap")
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "source": "nvml" if self._nv else "unavailable"}


# --------------------------------------------------------------------------- the arms
def cpu_oracle_rate(w, seed, budget_s=10.0, cap_s=30.0, sample_tokens=4096):
    """The fp64 oracle as it stands, on this host's cores, over a bounded sample of the workload:
    the first `sample_tokens` tokens of its (first) sequence, repeated until at least budget_s
    of CPU work has run (at least one copy)."""
    import oracle
    sample = min(sample_tokens, w.tokens)
    inp = inputs.prefill_inputs(w, seed, lengths=(sample,))
    dims = oracle.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    threads = oracle.default_threads()
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.prefill(dims, inp["x"], inp["beta"], inp["g"], inp["cu_seqlens"],
                       conv_w=inp["conv_w"], z=inp["z"], norm_w=inp["norm_w"], S0=inp["S0"],
                       nthreads=threads)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or el * (done + 1) / done > cap_s:
            break
    return {"value": done * sample / el, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} runs of the first {sample} tokens of {w.name} ({el:.1f} s)"}


def run_reference(args, w, seed, rank):
    """The fp64 CPU oracle as the reference arm, on this host's cores."""
    if rank != 0:
        return None
    import oracle
    # one step = a bounded sample of the workload: the first `sample` tokens of the sequence
    sample = 512
    inp = inputs.prefill_inputs(w, seed, lengths=(sample,))
    dims = oracle.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    threads = oracle.default_threads()

    def step():
        oracle.prefill(dims, inp["x"], inp["beta"], inp["g"], inp["cu_seqlens"],
                       conv_w=inp["conv_w"], z=inp["z"], norm_w=inp["norm_w"], nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = args.steps * sample / el
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": 1, "seq_len": w.tokens,
                   "sample_tokens_per_step": sample, "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{args.steps} steps of the first {sample} tokens"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def _graph_of(step):
    """The step's launches captured once as a CUDA graph (the library's trace, when attached,
    records each launch's events as event-record nodes of the graph)."""
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    return graph


def _kernel_table(per_step, T, w, peaks):
    """Per-kernel figures from the traced replays: per_step is a list (one per timed step) of
    [(name, ms)] launches.  Algorithmic work per step = per-token work x T; achieved = that work
    / the kernel's summed launch time per step (= work per launch / mean launch time for
    equal launches)."""
    fl, by = flops_per_token_by_kernel(w), bytes_per_token_by_kernel(w)
    kern = {}
    for recs in per_step:
        for name, ms in recs:
            k = kern.setdefault(name, {"launches": 0, "total_ms": 0.0})
            k["launches"] += 1
            k["total_ms"] += ms
    n = max(1, len(per_step))
    tot = sum(k["total_ms"] for k in kern.values()) or 1.0
    for name, k in kern.items():
        k["launches_per_step"] = k["launches"] / n
        k["ms_per_step"] = k["total_ms"] / n
        k["avg_ms"] = k["total_ms"] / k["launches"]
        k["share"] = k["total_ms"] / tot
        if name in fl:
            k["tflops"] = fl[name] * T / (k["ms_per_step"] * 1e-3) / 1e12
            k["tc_frac"] = k["tflops"] / peaks["bf16_tflops"]
            k["gbs"] = by[name] * T / (k["ms_per_step"] * 1e-3) / 1e9
            k["hbm_frac"] = k["gbs"] / peaks["hbm_gbs"]
    return kern


def _roofline(kern, T, peaks, peak_src, tokens_per_launch):
    """Roofline of the dominant kernel (largest time per step among the layer's kernels)."""
    cands = [k for k in kern if "tflops" in kern[k]]
    dom = max(cands, key=lambda k_: kern[k_]["ms_per_step"])
    dk = kern[dom]
    if dk["hbm_frac"] > dk["tc_frac"]:
        roof = {"bound": "hbm", "achieved": dk["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": dk["hbm_frac"]}
    else:
        roof = {"bound": "tensor", "achieved": dk["tflops"], "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": dk["tc_frac"]}
    tr = ncu_traffic(dom, tokens_per_launch)
    roof.update({"kernel": dom, "traffic": tr,
                 "traffic_note": "ncu dram read+write per launch, scaled from the capture's "
                                 "tokens to this launch's (profiles/traffic.json)"
                 if tr is not None else "null: no ncu capture of the current sources",
                 "peak_source": f"{peak_src} ({'burst bf16' if roof['bound'] == 'tensor' else 'copy'})"})
    return roof


def bench_prefill(args, w, seed, dev, gdn, peaks, peak_src, steps, warmup, e2e=True):
    """One prefill workload: CUDA-graph replays of the whole step (the step time), then as many
    replays of the step captured with the library's launch trace (per-kernel CUDA events of
    every replay), L2 flushed (256 MiB write, untimed) before each replay; optionally the
    end-to-end figure through the C ABI with host buffers."""
    import gated_deltanet_layer_02_b200 as _g  # noqa: F401  (the binding, already built)
    nvtx = torch.cuda.nvtx
    nvtx.range_push(f"prefill {w.name}: setup")
    inp = inputs.prefill_inputs(w, seed)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    dims = gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    T, N = w.tokens, len(w.lengths)
    out = torch.empty((T, w.num_v_heads, w.head_dim), dtype=w.dtype, device=dev)
    SN = torch.empty((N, w.num_v_heads, w.head_dim, w.head_dim), dtype=torch.float32, device=dev)
    convN = torch.empty((N, w.conv_kernel - 1, w.channels), dtype=w.dtype, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(N, T, w.dtype, dims), dtype=torch.uint8,
                     device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        gdn.chunk_prefill(d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"],
                          z=d["z"], norm_w=d["norm_w"], S0=d["S0"], SN=SN, convN=convN, out=out,
                          workspace=ws, dev_status=status, dims=dims)

    for _ in range(warmup):
        flush.zero_()
        step()
    nvtx.range_pop()

    def timed(graph, n_steps, tr=None):
        ms, per = [], []
        for _ in range(warmup):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize()
        for i in range(n_steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            b.synchronize()
            ms.append(a.elapsed_time(b))
            if tr is not None:
                per.append(tr.records())
        return ms, per

    # timed region: replays of the step's graph (the headline step time)
    graph = _graph_of(step)
    if dist_on():
        torch.distributed.barrier()
    torch.cuda.synchronize()
    nvtx.range_push(f"prefill {w.name}: timed")
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms, _ = timed(graph, steps)
    nvtx.range_pop()
    if dist_on():
        torch.distributed.barrier()
    del graph
    # the same step captured with the library's launch trace (an event pair around every launch,
    # recorded by each replay; launches in a traced capture go without programmatic dependent
    # launch), replayed as many times: the per-kernel times of the roofline
    nvtx.range_push(f"prefill {w.name}: traced")
    tr = gdn.Trace()
    with tr:
        tgraph = _graph_of(step)
    traced_ms, per_step = timed(tgraph, steps, tr)
    del tgraph
    tr.close()
    nvtx.range_pop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during the timed steps")
    res = {"workload": w.name, "tokens": T, "sequences": N, "step_ms": step_ms,
           "traced_graph_ms_per_step": statistics.mean(traced_ms),
           "launches_per_step": len(per_step[0]) if per_step else 0,
           "clocks": clk.summary()}
    nseg = max(1, sum(1 for n_, _ in per_step[0] if n_ == "gdn_prep")) if per_step else 1
    res["kernels"] = _kernel_table(per_step, T, w, peaks)
    res["roofline"] = _roofline(res["kernels"], T, peaks, peak_src, T / nseg)
    if e2e:
        nvtx.range_push(f"prefill {w.name}: e2e")
        res["e2e"] = _bench_e2e(args, w, inp, d, dims, dev, gdn, SN, convN, status, flush)
        nvtx.range_pop()
    return res


def _bench_e2e(args, w, inp, d, dims, dev, gdn, SN, convN, status, flush):
    """End to end through the C ABI with host buffers (gdn_chunk_prefill_host): the inputs'
    host->device copies, the layer and the output's device->host copy, overlapped segment by
    segment inside the call, all inside the timed region."""
    T, N = w.tokens, len(w.lengths)
    names = ("x", "beta", "g", "z")
    host = {k: inp[k].pin_memory() for k in names}
    out_h = torch.empty((T, w.num_v_heads, w.head_dim), dtype=w.dtype, pin_memory=True)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names) + inp["cu_seqlens"].numel() * 4
    d2h = out_h.numel() * out_h.element_size()
    cu_h = inp["cu_seqlens"]
    hws = torch.empty(gdn.lib().gdn_chunk_prefill_host_workspace_size(
        ctypes.byref(dims), ctypes.c_void_p(cu_h.data_ptr()), N, T, 0), dtype=torch.uint8,
        device=dev)
    e2e_ms = []
    reps = max(3, min(args.steps // 10, 20)) if T <= 65536 else 3
    for i in range(args.warmup + reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        a.record()
        gdn.chunk_prefill_host(host["x"], host["beta"], host["g"], cu_h, conv_w=d["conv_w"],
                               z=host["z"], norm_w=d["norm_w"], S0=d["S0"], SN=SN, convN=convN,
                               out=out_h, workspace=hws, dev_status=status, dims=dims)
        b.record()
        b.synchronize()
        if i >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the end-to-end steps")
    del hws, host, out_h
    return {"ms_per_step": statistics.mean(e2e_ms), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": reps}


def bench_chunk_states(args, w, seed, dev, gdn):
    """The prefill step with and without the chunk-boundary states (gdn_chunk_prefill_states),
    each timed as CUDA-graph replays with L2 flushed in between; extra bytes = the state writes."""
    inp = inputs.prefill_inputs(w, seed)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    dims = gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    T, N = w.tokens, len(w.lengths)
    C = sum((int(L) + 127) // 128 for L in w.lengths)
    cs = torch.empty((C, w.num_v_heads, w.head_dim, w.head_dim), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(N, T, w.dtype, dims), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((T, w.num_v_heads, w.head_dim), dtype=w.dtype, device=dev)
    SN = torch.empty((N, w.num_v_heads, w.head_dim, w.head_dim), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    res = {}
    for name, states in (("without", None), ("with", cs)):
        def step():
            gdn.chunk_prefill(d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"],
                              z=d["z"], norm_w=d["norm_w"], S0=d["S0"], SN=SN, out=out,
                              workspace=ws, dims=dims, chunk_states=states)
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        ms = []
        for _ in range(max(10, args.steps // 4)):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            graph.replay()
            b.record()
            b.synchronize()
            ms.append(a.elapsed_time(b))
        del graph
        res[name] = statistics.median(ms)
    return {"workload": w.name, "ms_per_step_without": res["without"],
            "ms_per_step_with": res["with"], "chunks": C,
            "extra_bytes_per_step": cs.numel() * 4}


def bench_block(w, seed, dev, gdn, hidden=2048, reps=20):
    """The token mixer (gdn_block_prefill: tcgen05 GEMM projections with the gates fused into the
    [b | a] projection, the layer, output
    projection) on the same sequences, hidden size 2048, eager calls with L2 flushed in between.
    flops_per_step counts the four projection GEMMs only."""
    bw = inputs.custom(w.num_k_heads, w.num_v_heads, w.head_dim, w.dtype, lengths=w.lengths)
    inp = inputs.block_inputs(bw, seed, hidden)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    dims = gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    T, N, Hv, dh = w.tokens, len(w.lengths), w.num_v_heads, w.head_dim
    y = torch.empty((T, hidden), dtype=w.dtype, device=dev)
    SN = torch.empty((N, Hv, dh, dh), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.lib().gdn_block_prefill_workspace_size(ctypes.byref(dims), hidden, N, T),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        gdn.block_prefill(d["h"], d["w_qkv"], d["w_z"], d["w_ba"], d["a_log"], d["dt_bias"],
                          d["w_out"], d["cu_seqlens"], conv_w=d["conv_w"], norm_w=d["norm_w"],
                          SN=SN, y=y, workspace=ws, dims=dims)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ms, per_kernel = [], {}
    tr = gdn.Trace()
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tr.reset()
        with tr:
            a.record()
            step()
            b.record()
        b.synchronize()
        ms.append(a.elapsed_time(b))
        for name, t_ in tr.records():
            per_kernel.setdefault(name, []).append(t_)
    tr.close()
    t = statistics.median(ms)
    C, HD = w.channels, Hv * dh
    gemm_flops = {"gemm_qkv": 2 * T * hidden * C, "gemm_z": 2 * T * hidden * HD,
                  "gemm_ba_gates": 2 * T * hidden * 2 * Hv, "gemm_out": 2 * T * HD * hidden}
    gemms = {}
    for name, f in gemm_flops.items():
        if name in per_kernel:
            k_ms = statistics.median(per_kernel[name])
            gemms[name] = {"ms": k_ms, "tflops": f / (k_ms * 1e-3) / 1e12}
    flops = sum(gemm_flops.values())
    return {"workload": f"{w.name}, hidden {hidden}", "ms_per_step": t,
            "tokens_per_s": T / (t * 1e-3), "projection_flops_per_step": flops,
            "gemms": gemms}


def bench_decode_multi(w, seed, dev, gdn, k=4, reps=20):
    """k tokens per sequence per call (speculative verification), fp32 state, no snapshots."""
    st = inputs.decode_state(w, seed)
    S, cs = st["S"].to(dev), st["conv_state"].to(dev)
    cw, nw = st["conv_w"].to(dev), st["norm_w"].to(dev)
    dims = gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    toks = [inputs.decode_step_inputs(w, seed, t) for t in range(k)]
    stk = {key: torch.stack([t[key] for t in toks], dim=1).contiguous().to(dev)
           for key in ("x", "beta", "g", "z")}
    out = torch.empty((w.batch, k, w.num_v_heads, w.head_dim), dtype=w.dtype, device=dev)
    call = lambda: gdn.decode_multi(stk["x"], stk["beta"], stk["g"], cs, S, cw, z=stk["z"],  # noqa: E731
                                    norm_w=nw, out=out, dims=dims)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        b.synchronize()
        ms.append(a.elapsed_time(b))
    m = statistics.median(ms)
    return m, 2 * S.numel() * 4, w.batch * k / (m * 1e-3)


def bench_decode(w, seed, dev, gdn, steps, state_dtype=torch.float32):
    st = inputs.decode_state(w, seed)
    S, cs = st["S"].to(dev).to(state_dtype), st["conv_state"].to(dev)
    cw, nw = st["conv_w"].to(dev), st["norm_w"].to(dev)
    dims = gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    steps_in = [{k: v.to(dev) for k, v in inputs.decode_step_inputs(w, seed, s).items()}
                for s in range(steps)]
    out = torch.empty((w.batch, w.num_v_heads, w.head_dim), dtype=w.dtype, device=dev)
    for s in steps_in[:3]:
        gdn.decode_step(s["x"], s["beta"], s["g"], cs, S, cw, z=s["z"], norm_w=nw, out=out,
                        dims=dims)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i, s in enumerate(steps_in):
            ev[i][0].record()
            gdn.decode_step(s["x"], s["beta"], s["g"], cs, S, cw, z=s["z"], norm_w=nw, out=out,
                            dims=dims)
            ev[i][1].record()
        torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    state_bytes = 2 * S.numel() * S.element_size()
    return statistics.median(ms), state_bytes, clk.summary()


def dist_on():
    return torch.distributed.is_available() and torch.distributed.is_initialized()


def max_over_ranks(values, device):
    """Element-wise maximum over ranks of per-rank times: the slowest rank sets the job's time."""
    if not dist_on():
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_s(world, tokens_per_rank, ms):
    """Whole-job throughput of weak-scaled replicas: all ranks' tokens over the slowest time."""
    return world * tokens_per_rank / (ms * 1e-3)


def profile_prefill(args, idx, dev, gdn):
    """The step graph of prefill workload `idx` replayed --warmup + --steps times (a small,
    self-contained command for ncu captures)."""
    w = inputs.CONFIGS[idx]
    inp = inputs.prefill_inputs(w, inputs.config_seed(idx))
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    dims = gdn.Dims(w.num_k_heads, w.num_v_heads, w.head_dim, w.conv_kernel)
    T, N = w.tokens, len(w.lengths)
    out = torch.empty((T, w.num_v_heads, w.head_dim), dtype=w.dtype, device=dev)
    SN = torch.empty((N, w.num_v_heads, w.head_dim, w.head_dim), dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.prefill_workspace_size(N, T, w.dtype, dims), dtype=torch.uint8,
                     device=dev)

    def step():
        gdn.chunk_prefill(d["x"], d["beta"], d["g"], d["cu_seqlens"], conv_w=d["conv_w"],
                          z=d["z"], norm_w=d["norm_w"], S0=d["S0"], SN=SN, out=out,
                          workspace=ws, dims=dims)
    ms = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        b.synchronize()
        if i >= args.warmup:
            ms.append(a.elapsed_time(b))
    return {"workload": w.name, "ms_per_step": statistics.mean(ms), "steps": args.steps}


#: the headline prefill workload (the largest single-GPU configuration: one 262,144-token
#: sequence) and the secondary prefill workloads reported beside it
HEADLINE = 4
SECONDARY = (1, 2)


def _prefill_line(res, n, peaks):
    """Whole-step figures of one prefill workload (max over ranks already applied to ms)."""
    T, ms = res["tokens"], res["ms_per_step"]
    w = inputs.CONFIGS[res["config_index"]]
    fl = flops_per_token_by_kernel(w)
    by = bytes_per_token_by_kernel(w)
    F = sum(v for k, v in fl.items())
    B = sum(v for k, v in by.items())
    value = job_tokens_per_s(n, T, ms)
    return value, {"tc_frac": F * value / n / (peaks["bf16_tflops"] * 1e12),
                   "hbm_frac": B * value / n / (peaks["hbm_gbs"] * 1e9),
                   "flops_per_token": F, "bytes_per_token": B, "chunk": CHUNK,
                   "flops_per_token_chunk64": sum(flops_per_token_by_kernel(w, 64).values())}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--headline-only", action="store_true",
                    help="only the headline prefill leg")
    ap.add_argument("--prefill-only", type=int, default=None, metavar="CONFIG",
                    help="profiling aid: only the step graph of prefill workload CONFIG (0-4), "
                         "--warmup + --steps replays, no other leg; prints its ms per step")
    ap.add_argument("--decode-only", action="store_true",
                    help="profiling aid: only the decode legs (fp32 state, bf16 state, 4-token "
                         "calls) of the decode workload, --decode-steps steps each")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = inputs.CONFIGS[HEADLINE]
    seed = inputs.config_seed(HEADLINE)
    if args.impl == "reference":
        res = run_reference(args, w, seed, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from gated_deltanet_layer_02_b200 import build as gdn_build
    gdn_build.build()
    import gated_deltanet_layer_02_b200 as gdn
    peaks, peak_src = load_peaks()
    n = world
    if args.prefill_only is not None:
        print(json.dumps(profile_prefill(args, args.prefill_only, dev, gdn)), flush=True)
        return
    if args.decode_only:
        w3, s3 = inputs.CONFIGS[3], inputs.config_seed(3)
        f32_ms = bench_decode(w3, s3, dev, gdn, args.decode_steps)[0]
        b16_ms = bench_decode(w3, s3, dev, gdn, args.decode_steps, torch.bfloat16)[0]
        multi_ms = bench_decode_multi(w3, s3, dev, gdn, reps=args.decode_steps)[0]
        print(json.dumps({"workload": w3.name, "decode_ms": f32_ms, "bf16_state_ms": b16_ms,
                          "multi_token_ms": multi_ms}), flush=True)
        return

    def run_prefill(idx, steps, e2e):
        r = bench_prefill(args, inputs.CONFIGS[idx], inputs.config_seed(idx), dev, gdn, peaks,
                          peak_src, steps, args.warmup, e2e=e2e)
        r["config_index"] = idx
        r["ms_per_step"], = max_over_ranks([statistics.mean(r.pop("step_ms"))], dev)
        if "e2e" in r:
            r["e2e"]["ms_per_step"], = max_over_ranks([r["e2e"]["ms_per_step"]], dev)
        return r

    head = run_prefill(HEADLINE, args.steps, True)
    value, step_roof = _prefill_line(head, n, peaks)
    T = head["tokens"]
    others = {}
    if not args.headline_only:
        for idx in SECONDARY:
            r = run_prefill(idx, max(20, args.steps), False)
            v, sr = _prefill_line(r, n, peaks)
            r.update({"value": v, "unit": "tokens/s", "step_roofline": sr})
            others[r["workload"]] = r
    head_e2e = head.pop("e2e")
    e2e = {"value": job_tokens_per_s(n, T, head_e2e["ms_per_step"]), "unit": "tokens/s",
           "ms_per_step": head_e2e["ms_per_step"], "steps": head_e2e["steps"],
           "h2d_bytes_per_step": head_e2e["h2d_bytes_per_step"],
           "d2h_bytes_per_step": head_e2e["d2h_bytes_per_step"],
           "path": "gdn_chunk_prefill_host (C ABI, pinned host buffers, copies overlapped with "
                   "the layer segment by segment)"}

    decode = None
    chunk_states = block = None
    if not args.headline_only:
        torch.cuda.nvtx.range_push("decode")
        dec_ms, dec_bytes, dec_clk = bench_decode(inputs.CONFIGS[3], inputs.config_seed(3), dev,
                                                  gdn, args.decode_steps)
        dec_ms = max_over_ranks([dec_ms], dev)[0]
        dec_gbs = n * dec_bytes / (dec_ms * 1e-3) / 1e9
        # the serving option of a bf16 recurrent state (same workload, half the state bytes)
        d16_ms, d16_bytes, d16_clk = bench_decode(inputs.CONFIGS[3], inputs.config_seed(3), dev,
                                                  gdn, args.decode_steps, torch.bfloat16)
        d16_ms = max_over_ranks([d16_ms], dev)[0]
        d16_gbs = n * d16_bytes / (d16_ms * 1e-3) / 1e9
        dm_ms, dm_bytes, dm_tps = bench_decode_multi(inputs.CONFIGS[3], inputs.config_seed(3),
                                                     dev, gdn)
        dm_ms = max_over_ranks([dm_ms], dev)[0]
        torch.cuda.nvtx.range_pop()
        decode = {"workload": inputs.CONFIGS[3].name, "value": dec_gbs, "unit": "GB/s",
                  "ms_per_step": dec_ms, "steps": args.decode_steps,
                  "roofline": {"bound": "hbm", "achieved": dec_gbs / n, "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": dec_gbs / n / peaks["hbm_gbs"],
                               "traffic": ncu_traffic("decode_step"),
                               "peak_source": f"{peak_src} (copy)"},
                  "clocks": dec_clk,
                  "bf16_state": {"value": d16_gbs, "unit": "GB/s", "ms_per_step": d16_ms,
                                 "sequence_steps_per_s": n * inputs.CONFIGS[3].batch / (d16_ms * 1e-3),
                                 "roofline": {"bound": "hbm", "achieved": d16_gbs / n,
                                              "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                              "frac": d16_gbs / n / peaks["hbm_gbs"],
                                              "traffic": ncu_traffic("decode_step_bf16_state"),
                                              "peak_source": f"{peak_src} (copy)"},
                                 "clocks": d16_clk},
                  "multi_token": {"tokens_per_call": 4, "ms_per_call": dm_ms,
                                  "sequence_tokens_per_s": n * inputs.CONFIGS[3].batch * 4 / (dm_ms * 1e-3),
                                  "one_token_steps_ms": 4 * dec_ms,
                                  "state_gbs": n * dm_bytes / (dm_ms * 1e-3) / 1e9,
                                  "roofline": {"bound": "hbm",
                                               "achieved": dm_bytes / (dm_ms * 1e-3) / 1e9,
                                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                               "frac": dm_bytes / (dm_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                               "traffic": ncu_traffic("decode_multi"),
                                               "peak_source": f"{peak_src} (copy)"}}}
        w1 = inputs.CONFIGS[1]
        chunk_states = bench_chunk_states(args, w1, inputs.config_seed(1), dev, gdn)
        block = bench_block(w1, inputs.config_seed(1), dev, gdn)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_rate(w, seed)

    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; Qwen3-Next GDN layer shapes)",
        "config": {"workload": w.name, "global_batch": n, "seq_len": T,
                   "parallelism": "replicas" if n == 1 else f"replicas x{n}",
                   "l2": "flushed between timed steps (256 MiB write, untimed); inputs 8.7 GB "
                         "> L2 as well",
                   "launch": "CUDA graph replay of the whole step; per-kernel times from as many "
                             "replays of the same step captured with the library's launch trace "
                             "(event-record nodes around every launch)",
                   "chunk": CHUNK, "heads": [w.num_k_heads, w.num_v_heads], "head_dim": 128},
        "roofline": head["roofline"], "step_roofline": step_roof, "kernels": head["kernels"],
        "traced_graph_ms_per_step": head["traced_graph_ms_per_step"],
        "e2e": e2e, "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": head["clocks"], "prefill_configs": others, "decode": decode,
        "chunk_states": chunk_states, "block": block, "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist_on():
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
