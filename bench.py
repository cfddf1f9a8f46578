"""Benchmark of the gated delta-rule forward pass on B200.

One step = one pass of the whole hot path over one batch: the chunkwise
prefill (cumulative gate, UT transform, state pass, output) of the FG2-GDN+
workload -- the largest single-GPU configuration (B=1, H=32, T=32768,
dk=dv=128, chunk 64, bf16 q/k/v, channel-wise alpha, beta_k and beta_v, fp32
state) -- then one recurrent decode step that continues every (b, h) from the
prefill's final state (prefill -> decode handoff).  That step is the headline
value.  The same run times the prefill of every other workload (KDA/FG2-GDN,
Gated DeltaNet, fp32 DeltaNet), each with its own roofline, and the
memory-bound decode workload (B=256, H=32, 512 MiB fp32 state, chained
in-place steps), reported under "workloads" and "decode".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With N > 1 launch under torch.distributed.run: every rank runs its own batch
(heads are independent: weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

from synth import CONFIGS, DECODE, decode_inputs, make_inputs, problem

METRIC = "delta-rule fwd Mtokens·heads/s (prefill) & decode GB/s; % of roofline"
HOST_COVER_CYCLES = 400_000  # about 0.2 ms of GPU sleep ahead of a timed launch that follows an L2 flush
WORKLOAD = "fg2plus_bf16"  # the headline step's workload: the largest single-GPU configuration
PREFILL_WORKLOADS = ("fg2plus_bf16", "kda_bf16", "gdn_bf16", "deltanet_f32")
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- work model
def flops_per_token_head(dk, dv, C):
    """Algorithmic FLOPs of the chunkwise form per token and head (triangular masks exploited)."""
    return C * (3 * dk + 2 * dv) + 6 * dk * dv + C * C / 3.0


def prefill_bytes(p, with_S0):
    """Algorithmic HBM bytes of one prefill: inputs read once, outputs written once."""
    io = 2 if p.io == "bf16" else 4
    per = io * (2 * p.dk + 2 * p.dv)
    per += {"none": 0, "scalar": 4, "channel": 4 * p.dk}[p.alpha]
    per += {"scalar": 4, "channel": 4 * p.dk}[p.beta_k]
    per += {"none": 0, "scalar": 4, "channel": 4 * p.dv}[p.beta_v]
    state = p.B * p.H * p.dk * p.dv * 4 * (2 if with_S0 else 1)
    return p.token_heads * per + state


def decode_bytes(B, H, dk, dv, io=2, alpha_ch=True, beta_ch=True):
    """Per decode step: state read + write, q, k, v, o, gates."""
    heads = B * H
    per = 2 * dk * dv * 4 + io * (2 * dk + 2 * dv) + (4 * dk if alpha_ch else 4) + (4 * dk if beta_ch else 4)
    return heads * per


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the ncu captures
# summarised under profiles/, each valid only for the kernel sources it was taken on: the key is
# a digest of the kernel's own source files under csrc/ (see csrc_digest), so any change to them
# voids the number, and the workload it was taken on, so other workloads report none.  Captures on
# a shorter sequence of the same workload (T noted in the profile) are scaled by T to a full launch.
RING_SOURCES = ("chunk_tc3.cuh", "chunk_tc.cuh", "tri_inverse.cuh", "sm100.cuh", "common.cuh")
QUAD_SOURCES = ("chunk_tc4.cuh", "chunk_tc.cuh", "tri_inverse.cuh", "sm100.cuh", "common.cuh")
BWD_CHUNK_SOURCES = ("backward_chunk.cuh",) + RING_SOURCES
MEASURED_TRAFFIC = {
    ("chunk_fwd_ring_kernel", "gdn_bf16"): ("c4c8aa6942ac", 249.20e6, RING_SOURCES),
    ("chunk_fwd_ring_kernel", "kda_bf16"): ("c4c8aa6942ac", 530.25e6, RING_SOURCES),
    ("chunk_fwd_ring_kernel", "fg2plus_bf16"): ("c4c8aa6942ac", 4 * 663.67e6, RING_SOURCES),  # T = 8192 x 4
    ("chunk_fwd_quad_kernel", "kda_bf16"): ("1b1675a62aab", 537.56e6, QUAD_SOURCES),
    ("chunk_fwd_quad_kernel", "fg2plus_bf16"): ("1b1675a62aab", 4 * 674.51e6, QUAD_SOURCES),  # T = 8192 x 4
    ("chunk_fwd_simt_kernel", "deltanet_f32"): ("31898eacf605", 0.4628e6, ("chunk_simt.cuh", "common.cuh")),
    ("decode_stream_kernel", "decode_bf16"): ("6cb82d40c1fd", 1031.005696e6, ("decode_stream.cuh", "common.cuh")),
    ("delta_rule_bwd_kernel", "gdn_bf16"): ("9a0d1d786d6e", 10536.615e6, ("backward.cuh", "common.cuh")),
    ("chunk_bwd_kernel", "gdn_bf16"): ("b945780a1cf8", 4 * 207.81e6, BWD_CHUNK_SOURCES),  # T = 1024 x 4
}

def decode_kernel_name(heads, sms=148):
    """The decode kernel the library runs for dk = dv = 128: the persistent streaming kernel for
    more heads than SMs, else four CTAs per head."""
    return "decode_stream_kernel" if heads > sms else "decode_step_kernel"


def prefill_kernel_name(p, ws_bytes=256):
    """The prefill kernel the library runs for a problem (the dispatch of dr_chunk_fwd).  For the
    cluster shapes, the library asks for factor staging in the workspace (dr_chunk_fwd_workspace
    above the 256-byte status word) exactly when it runs the four-CTA kernel."""
    if p.io == "bf16" and p.dk == 128 and p.chunk == 64:
        if p.dv != 128:
            return "chunk_fwd_tc_kernel"
        return "chunk_fwd_quad_kernel" if ws_bytes > 256 else "chunk_fwd_ring_kernel"
    return "chunk_fwd_simt_kernel"


def csrc_digest(only=None):
    """sha1 over the kernel sources (all of csrc/, or the files named in `only`), in name order."""
    import hashlib

    d = os.path.join(ROOT, "weight_recurrence_chunkwise_b200", "csrc")
    h = hashlib.sha1()
    for name in sorted(os.listdir(d)):
        if only is not None and name not in only:
            continue
        with open(os.path.join(d, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(kernel, workload):
    """Bytes per launch from the committed ncu summary, or None once the kernel sources changed."""
    if (kernel, workload) not in MEASURED_TRAFFIC:
        return None
    prefix, nbytes, only = MEASURED_TRAFFIC[(kernel, workload)]
    try:
        digest = csrc_digest(only)
    except OSError:
        return None
    return nbytes if digest.startswith(prefix) else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index, period=0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, ws, device):
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_problem(rank, workload=WORKLOAD):
    """The workload a rank runs: same shape, its own seed (heads are independent, no exchange)."""
    base = CONFIGS[workload]
    return base.replace(seed=base.seed + 1000 * rank)


def to_dev(x, dev):
    return {k: (None if t is None else t.to(dev)) for k, t in x.items()}


def oracle_sample(p, threads):
    """A bounded sample of a workload for the float64 oracle: whole heads (all T), about one long
    head per host thread (at most the whole batch) -- some 10-30 s of CPU work at most."""
    heads_per_thread = max(1, round(4096 * 4 / p.T))
    want = max(1, min(p.B * p.H, heads_per_thread * threads))
    H = min(p.H, want)
    B = max(1, min(p.B, want // H))
    return p.replace(B=B, H=H)


def cpu_oracle_sample(p):
    """Time the float64 oracle on a bounded sample of the workload, all host cores, plus one head on
    one thread for the per-core rate."""
    import oracle

    threads = oracle.max_threads()
    x = make_inputs(oracle_sample(p, threads))
    t0 = time.perf_counter()
    oracle.delta_rule_sequential(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], beta_v=x["beta_v"],
                                 S0=x["S0"], threads=threads)
    dt = time.perf_counter() - t0
    th = x["q"].shape[0] * x["q"].shape[1] * x["q"].shape[2]
    # one thread on one whole head, for the per-core rate
    x1 = {k: (None if t is None else (t[:1, :, :1] if k != "S0" else t[:1, :1])) for k, t in x.items()}
    t1 = time.perf_counter()
    oracle.delta_rule_sequential(x1["q"], x1["k"], x1["v"], x1["beta_k"], alpha=x1["alpha"], beta_v=x1["beta_v"],
                                 S0=x1["S0"], threads=1)
    dt1 = time.perf_counter() - t1
    return {"value": th / dt / 1e6, "unit": "Mtokens·heads/s", "cores": threads, "kind": "oracle",
            "hardware_concurrency": os.cpu_count(), "single_thread_value": p.T / dt1 / 1e6,
            "sample": f"{x['q'].shape[0] * x['q'].shape[2]} whole heads x T={p.T} of the {p.name} workload, float64, "
                      f"{threads} OpenMP threads, {dt:.2f} s; single thread: one head, {dt1:.2f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, ws, rank):
    """The reference arm: the float64 oracle as it stands, timed on the host cores, each step a
    bounded sample (whole heads) of the headline workload.  Rank 0 only."""
    if rank != 0:
        return 0
    import oracle

    p = CONFIGS[WORKLOAD]
    threads = oracle.max_threads()
    sub = oracle_sample(p, threads)
    sample_heads = sub.B * sub.H
    xs = make_inputs(sub)
    run = lambda: oracle.delta_rule_sequential(xs["q"], xs["k"], xs["v"], xs["beta_k"], alpha=xs["alpha"],
                                               beta_v=xs["beta_v"], S0=xs["S0"], threads=threads)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    th = sample_heads * p.T
    v = th / dt / 1e6
    sample = f"{sample_heads} whole heads x T={p.T} of {p.name} per step, float64 oracle, {threads} threads"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "Mtokens·heads/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": p.name, "B": p.B, "H": p.H, "T": p.T, "dk": p.dk, "dv": p.dv, "chunk": p.chunk},
            "cpu_baseline": {"value": v, "unit": "Mtokens·heads/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "Mtokens·heads/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_decode_only(args, dr, dev, st, ws):
    """Profiling aid: the decode workload alone (warm-up, then the timed chained steps)."""
    d = decode_inputs()
    S_dec = d["S"].to(dev)
    pool = {k: (None if d[k] is None else d[k].to(dev)) for k in ("q", "k", "v", "alpha", "beta_k")}
    o_dec = torch.empty((DECODE.B, 1, DECODE.H, DECODE.dv), dtype=torch.bfloat16, device=dev)
    n = args.warmup + args.decode_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(n):
        if i == args.warmup:
            e0.record(st)
        j = i % DECODE.pool
        dr.dr_decode_step(pool["q"][j], pool["k"][j], pool["v"][j], pool["beta_k"][j], S_dec,
                          alpha=pool["alpha"][j], o=o_dec, stream=st)
    e1.record(st)
    torch.cuda.synchronize()
    dms = e0.elapsed_time(e1) / args.decode_steps
    dgbs = decode_bytes(DECODE.B, DECODE.H, DECODE.dk, DECODE.dv) / (dms / 1e3) / 1e9
    print(json.dumps({"only_decode": True, "ms_per_step": dms, "GB/s": dgbs}), flush=True)
    return 0


def backward_bytes(p):
    """Algorithmic HBM bytes of one backward: q, k, v, dout, gates, S0, dS_T read; fp32 gradients written."""
    io = 2 if p.io == "bf16" else 4
    gate = lambda m, w: {"none": 0, "scalar": 4, "channel": 4 * w}[m]
    per_in = io * (2 * p.dk + 2 * p.dv) + gate(p.alpha, p.dk) + gate(p.beta_k, p.dk) + gate(p.beta_v, p.dv)
    per_out = 4 * (2 * p.dk + p.dv) + gate(p.alpha, p.dk) + gate(p.beta_k, p.dk) + gate(p.beta_v, p.dv)
    state = p.B * p.H * p.dk * p.dv * 4
    return p.token_heads * (per_in + per_out) + 3 * state


def run_backward(args, dr, p, x, dev, st, peaks, peaks_src):
    """Profiling aid: the backward pass alone on one workload (warm-up, then timed launches), through
    the library's choice of kernel and, for comparison, the token-sequential kernel."""
    g = torch.Generator().manual_seed(p.seed)
    dout = torch.randn(x["v"].shape, generator=g).to(x["v"].dtype).to(dev)
    S0 = torch.zeros((p.B, p.H, p.dk, p.dv), dtype=torch.float32, device=dev)
    dST = torch.randn((p.B, p.H, p.dk, p.dv), generator=g).to(dev)
    chunk_path = p.io == "bf16" and p.dk == 128 and p.dv == 128
    out = {"backward": True, "workload": p.name, "T": p.T}
    for variant in (["default", "sequential"] if chunk_path else ["default"]):
        run = lambda: dr.dr_diag_backward_variant(variant, x["q"], x["k"], x["v"], x["beta_k"], dout,
                                                  alpha=x["alpha"], beta_v=x["beta_v"], S0=S0, dS_T=dST, stream=st)
        for _ in range(args.warmup):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(args.steps):
            run()
        e1.record(st)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        byts = backward_bytes(p)
        gbs = byts / (ms / 1e3) / 1e9
        chunked = variant == "default" and chunk_path
        kern = "chunk_fwd_ring_kernel (states) + chunk_bwd_kernel" if chunked else "delta_rule_bwd_kernel"
        out["sequential" if variant == "sequential" else "ms_kernel"] = kern
        out[variant] = {"ms": ms, "kernel": kern,
                        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": gbs / peaks["hbm_gbs"], "peak_source": peaks_src,
                                     "traffic": None if chunked else measured_traffic("delta_rule_bwd_kernel", p.name),
                                     "algorithmic_bytes_per_launch": byts}}
        if chunked:  # the two launches' own DRAM traffic (forward with chunk states, then the backward walk)
            out[variant]["traffic_by_kernel"] = {
                "chunk_fwd_ring_kernel": None,  # with states stored: not captured
                "chunk_bwd_kernel": measured_traffic("chunk_bwd_kernel", p.name) if p.T == CONFIGS[p.name].T else None}
    print(json.dumps(out), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def prefill_roofline(p, ms, peaks, peaks_src, with_S0=False, ws_bytes=256, variant="default"):
    """Roofline of one prefill launch: HBM-bound on algorithmic counts (SURVEY-style work model)."""
    byts = prefill_bytes(p, with_S0=with_S0)
    flops = p.token_heads * flops_per_token_head(p.dk, p.dv, p.chunk)
    gbs = byts / (ms / 1e3) / 1e9
    t_roof_ms = max(byts / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops_sustained"] * 1e12)) * 1e3
    kern = {"ring": "chunk_fwd_ring_kernel", "quad": "chunk_fwd_quad_kernel"}.get(variant) or prefill_kernel_name(p, ws_bytes)
    return {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
            "traffic": measured_traffic(kern, p.name), "peak_source": peaks_src, "kernel": kern,
            "algorithmic_bytes_per_launch": byts, "algorithmic_flops_per_launch": flops,
            "tensor_tflops_achieved": flops / (ms / 1e3) / 1e12, "roofline_time_ms": t_roof_ms,
            "frac_of_max_roofline": t_roof_ms / ms}


def time_prefill_workload(dr, p, dev, st, steps, warmup, ws, peaks, peaks_src, variant="default"):
    """Prefill alone on one workload: mean CUDA-event duration of each launch, max over ranks.

    Inputs larger than L2 need no flush; a smaller workload gets an L2 flush (a 256 MiB write)
    between launches, outside the per-launch events.  `variant` names a kernel of
    dr_diag_chunk_fwd_variant instead of the library's choice (a profiling aid)."""
    x = to_dev(make_inputs(p), dev)
    o = torch.empty_like(x["v"])
    S = torch.empty((p.B, p.H, p.dk, p.dv), dtype=torch.float32, device=dev)
    prob = dr.make_problem(x["q"], x["v"], x["alpha"], x["beta_k"], x["beta_v"], p.chunk)
    if variant == "default":
        need = dr.workspace_bytes(prob)
    else:
        need = int(dr.lib().dr_diag_chunk_fwd_workspace(dr.PREFILL_VARIANTS[variant], ctypes.byref(prob)))
    wsb = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    in_bytes = sum(t.numel() * t.element_size() for t in x.values() if t is not None)
    flush = None if in_bytes > L2_BYTES else torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    if variant == "default":
        run = lambda: dr.dr_chunk_fwd(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], beta_v=x["beta_v"],
                                      S0=x["S0"], chunk=p.chunk, o=o, S_T=S, workspace=wsb, stream=st)
    else:
        run = lambda: dr.dr_diag_chunk_fwd_variant(variant, x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"],
                                                   beta_v=x["beta_v"], S0=x["S0"], chunk=p.chunk, o=o, S_T=S,
                                                   workspace=wsb, stream=st)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    if dr.dr_workspace_status(wsb) != dr.DR_OK:
        raise RuntimeError(f"{p.name}: device status {dr.dr_workspace_status(wsb)}")
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(mk(), mk()) for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize()
    for e0, e1 in ev:
        if flush is not None:
            with torch.cuda.stream(st):
                flush.fill_(1)
                # keep the stream busy while the host enqueues the launch, so that the events time the
                # kernel and not the host's launch latency
                torch.cuda._sleep(HOST_COVER_CYCLES)
        e0.record(st)
        run()
        e1.record(st)
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev), ws, dev)
    return {"workload": p.name, "B": p.B, "H": p.H, "T": p.T, "dk": p.dk, "dv": p.dv, "chunk": p.chunk,
            "io": p.io, "alpha": p.alpha, "beta_k": p.beta_k, "beta_v": p.beta_v, "S0": p.S0,
            "ms": ms, "value": p.token_heads * ws / (ms / 1e3) / 1e6, "unit": "Mtokens·heads/s", "launches": steps,
            "l2": "inputs larger than L2, no flush" if flush is None else "L2 flushed (256 MiB write) between launches",
            "roofline": prefill_roofline(p, ms, peaks, peaks_src, with_S0=x["S0"] is not None, ws_bytes=need,
                                         variant=variant)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000,
                    help="chained in-place decode steps timed (the decode workload is 1000 steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--serial-steps", action="store_true",
                    help="run each step's handoff decode after its prefill on one stream (no overlap of steps)")
    ap.add_argument("--only-prefill", action="store_true",
                    help="profiling aid: time only the prefill of the --config workload")
    ap.add_argument("--only-decode", action="store_true",
                    help="profiling aid: time only the decode workload")
    ap.add_argument("--config", default=WORKLOAD, choices=list(CONFIGS),
                    help="with --only-prefill / --backward: the workload to time (default: the headline one)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (dr_backward) on the --config workload instead")
    ap.add_argument("--prefill-variant", default="default", choices=["default", "ring", "quad"],
                    help="with --only-prefill: time the named cluster kernel instead of the library's choice")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="with --only-prefill / --backward: override the workload's T (profiling a shorter case "
                         "of the same shape; the line reports the T it ran)")
    ap.add_argument("--seqpar-cost", action="store_true",
                    help="time one rank's work of a sequence-parallel prefill of the --config workload split "
                         "over 2, 4 and 8 ranks (on this one GPU) beside the unsplit prefill")
    args = ap.parse_args()
    ws, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, ws, rank)
    args.warmup = max(args.warmup, 3)

    import weight_recurrence_chunkwise_b200 as dr

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    peaks, peaks_src = load_peaks()
    st = torch.cuda.current_stream()

    if args.only_decode:
        return run_decode_only(args, dr, dev, st, ws)
    def aid_problem():  # the workload of a profiling aid, with its T overridden if asked
        p = rank_problem(rank, args.config)
        return p if args.seq_len is None else p.replace(T=args.seq_len)

    if args.backward:
        p = aid_problem()
        return run_backward(args, dr, p, to_dev(make_inputs(p), dev), dev, st, peaks, peaks_src)
    if args.seqpar_cost:
        return run_seqpar_cost(args, dr, rank_problem(rank, args.config), dev, st)
    if args.only_prefill:
        line = time_prefill_workload(dr, aid_problem(), dev, st, args.steps, args.warmup, ws, peaks, peaks_src,
                                     variant=args.prefill_variant)
        if rank == 0:
            print(json.dumps({"only_prefill": True, "prefill_ms": line["ms"], **line}), flush=True)
        return 0

    # ---------------- every prefill workload on its own (each rank its own seeded batch)
    workloads = {}
    for name in PREFILL_WORKLOADS:
        if name == WORKLOAD:
            continue  # timed below as the headline step
        workloads[name] = time_prefill_workload(dr, rank_problem(rank, name), dev, st, args.steps, args.warmup, ws,
                                                peaks, peaks_src)
        torch.cuda.empty_cache()

    # ---------------- the headline step: prefill of the headline workload -> one decode step
    p = rank_problem(rank, WORKLOAD)
    x = to_dev(make_inputs(p), dev)
    nxt = to_dev(make_inputs(p.replace(T=1, seed=p.seed + 500)), dev)  # the token after the prompt
    o = torch.empty_like(x["v"])
    S = torch.empty((p.B, p.H, p.dk, p.dv), dtype=torch.float32, device=dev)
    o1 = torch.empty_like(nxt["v"])
    ws_buf = torch.zeros(max(dr.workspace_bytes(dr.make_problem(x["q"], x["v"], x["alpha"], x["beta_k"],
                                                                 x["beta_v"], p.chunk)), 256),
                         dtype=torch.uint8, device=dev)

    def step():
        dr.dr_chunk_fwd(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], beta_v=x["beta_v"], S0=None,
                        chunk=p.chunk, o=o, S_T=S, workspace=ws_buf, stream=st)
        dr.dr_decode_step(nxt["q"], nxt["k"], nxt["v"], nxt["beta_k"], S, alpha=nxt["alpha"], beta_v=nxt["beta_v"],
                          o=o1, stream=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dr.dr_workspace_status(ws_buf) == dr.DR_OK

    n = args.steps
    # Steps are pipelined unless --serial-steps: step i's handoff decode runs on a second stream
    # beside step i+1's prefill (which leaves SMs free), with the final state double-buffered; the
    # prefill's stream has the higher priority.  Every step still does all of its work inside the
    # timed region.
    pipelined = not args.serial_steps
    pf = torch.cuda.Stream(device=dev, priority=-1) if pipelined else st
    dec = torch.cuda.Stream(device=dev) if pipelined else st
    S_buf = [S, torch.empty_like(S)] if pipelined else [S, S]
    o1_buf = [o1, torch.empty_like(o1)] if pipelined else [o1, o1]
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(mk(), mk(), mk(), mk()) for _ in range(n)]  # prefill start / end, decode start / end
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_start, t_end = mk(), mk()
        t_start.record(pf)
        if dec is not pf:
            dec.wait_event(t_start)
        for i in range(n):
            j = i % 2
            if pipelined and i >= 2:
                pf.wait_event(ev[i - 2][3])  # the decode of step i-2 is done with S_buf[j]
            ev[i][0].record(pf)
            dr.dr_chunk_fwd(x["q"], x["k"], x["v"], x["beta_k"], alpha=x["alpha"], beta_v=x["beta_v"], S0=None,
                            chunk=p.chunk, o=o, S_T=S_buf[j], workspace=ws_buf, stream=pf)
            ev[i][1].record(pf)
            if dec is not pf:
                dec.wait_event(ev[i][1])
            ev[i][2].record(dec)
            dr.dr_decode_step(nxt["q"], nxt["k"], nxt["v"], nxt["beta_k"], S_buf[j], alpha=nxt["alpha"],
                              beta_v=nxt["beta_v"], o=o1_buf[j], stream=dec)
            ev[i][3].record(dec)
        if dec is not pf:
            pf.wait_stream(dec)
        t_end.record(pf)
        torch.cuda.synchronize()
    barrier(ws)
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), ws, dev)
    ms_step = ms_total / n
    prefill_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[1]) for e in ev), ws, dev)
    handoff_ms = max_over_ranks(statistics.mean(e[2].elapsed_time(e[3]) for e in ev), ws, dev)
    tok_heads = p.B * p.H * (p.T + 1)
    value = tok_heads * ws / (ms_step / 1e3) / 1e6
    roofline = prefill_roofline(p, prefill_ms, peaks, peaks_src, ws_bytes=ws_buf.numel())
    workloads[WORKLOAD] = {"workload": p.name, "B": p.B, "H": p.H, "T": p.T, "dk": p.dk, "dv": p.dv,
                           "chunk": p.chunk, "ms": prefill_ms, "value": p.token_heads * ws / (prefill_ms / 1e3) / 1e6,
                           "unit": "Mtokens·heads/s", "launches": n, "l2": "inputs larger than L2, no flush",
                           "roofline": roofline, "note": "prefill launches of the headline step"}

    # ---------------- decode workload (B=256, H=32, 512 MiB state, chained in-place steps)
    d = decode_inputs()
    S_dec = d["S"].to(dev)
    pool = {k: (None if d[k] is None else d[k].to(dev)) for k in ("q", "k", "v", "alpha", "beta_k")}
    o_dec = torch.empty((DECODE.B, 1, DECODE.H, DECODE.dv), dtype=torch.bfloat16, device=dev)
    del d

    def dstep(i):
        j = i % DECODE.pool
        dr.dr_decode_step(pool["q"][j], pool["k"][j], pool["v"][j], pool["beta_k"][j], S_dec, alpha=pool["alpha"][j],
                          o=o_dec, stream=st)

    for i in range(3):
        dstep(i)
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(args.decode_steps):
        dstep(i)
    e1.record(st)
    torch.cuda.synchronize()
    dms = max_over_ranks(e0.elapsed_time(e1), ws, dev) / args.decode_steps
    dbytes = decode_bytes(DECODE.B, DECODE.H, DECODE.dk, DECODE.dv)
    dgbs = dbytes / (dms / 1e3) / 1e9

    # the same chained steps captured in a CUDA graph (one pool cycle per graph) and replayed
    cap = torch.cuda.Stream()
    cap.wait_stream(st)

    def dstep_on(i, stream):
        j = i % DECODE.pool
        dr.dr_decode_step(pool["q"][j], pool["k"][j], pool["v"][j], pool["beta_k"][j], S_dec, alpha=pool["alpha"][j],
                          o=o_dec, stream=stream)

    with torch.cuda.stream(cap):
        for i in range(3):
            dstep_on(i, cap)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        for i in range(DECODE.pool):
            dstep_on(i, cap)
    reps = max(1, args.decode_steps // DECODE.pool)
    torch.cuda.synchronize()
    barrier(ws)
    e0.record(st)
    for _ in range(reps):
        graph.replay()
    e1.record(st)
    torch.cuda.synchronize()
    dms_graph = max_over_ranks(e0.elapsed_time(e1), ws, dev) / (reps * DECODE.pool)
    del graph
    dheads = DECODE.B * DECODE.H
    decode = {"value": dgbs * ws, "unit": "GB/s", "ms_per_step": dms, "steps": args.decode_steps,
              "graph": {"ms_per_step": dms_graph, "GB/s": dbytes / (dms_graph / 1e3) / 1e9 * ws,
                        "steps": reps * DECODE.pool},
              "config": {"workload": DECODE.name, "B": DECODE.B, "H": DECODE.H, "dk": DECODE.dk, "dv": DECODE.dv,
                         "state_MiB": DECODE.B * DECODE.H * DECODE.dk * DECODE.dv * 4 / 2 ** 20},
              "roofline": {"bound": "hbm", "achieved": dgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": dgbs / peaks["hbm_gbs"],
                           "traffic": measured_traffic(decode_kernel_name(dheads), DECODE.name),
                           "peak_source": peaks_src,
                           "kernel": decode_kernel_name(dheads), "algorithmic_bytes_per_launch": dbytes}}
    del S_dec, pool

    # ---------------- end to end through the public API with host buffers (pinned), copies timed.
    # Steps are pipelined over two buffer slots and three streams, as a caller streaming batches
    # would: step i's host->device copies overlap step i-1's kernels and step i-2's device->host
    # copies (PCIe carries both directions at once).  Every step still moves all its inputs in and
    # all its results out inside the timed region.
    host = {k: (None if t is None else t.cpu().pin_memory()) for k, t in x.items()}
    host_n = {k: (None if t is None else t.cpu().pin_memory()) for k, t in nxt.items()}
    h2d = sum(t.numel() * t.element_size() for t in list(host.values()) + list(host_n.values()) if t is not None)
    d2h = o.numel() * o.element_size() + S.numel() * 4 + o1.numel() * o1.element_size()
    e2e_steps = max(3, min(6, n))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    dev_like = lambda h: {k: (None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev))
                          for k, t in h.items()}
    slots = [{"g": dev_like(host), "gn": dev_like(host_n), "o": torch.empty_like(o), "S": torch.empty_like(S),
              "o1": torch.empty_like(o1), "o_h": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
              "S_h": torch.empty(S.shape, dtype=S.dtype).pin_memory(),
              "o1_h": torch.empty(o1.shape, dtype=o1.dtype).pin_memory(),
              "in": torch.cuda.Event(), "done": torch.cuda.Event(), "out": torch.cuda.Event()} for _ in range(2)]
    for sl in slots:  # every event recorded once, so the first waits on it are satisfied
        for e in ("in", "done", "out"):
            sl[e].record(st)

    def e2e_step(i):
        sl = slots[i % 2]
        s_in.wait_event(sl["done"])  # step i-2's kernels no longer read this slot's inputs
        with torch.cuda.stream(s_in):
            for src, dst in ((host, sl["g"]), (host_n, sl["gn"])):
                for k, t in src.items():
                    if t is not None:
                        dst[k].copy_(t, non_blocking=True)
        sl["in"].record(s_in)
        st.wait_event(sl["in"])
        st.wait_event(sl["out"])  # step i-2's results have been read back
        g, gn = sl["g"], sl["gn"]
        dr.dr_chunk_fwd(g["q"], g["k"], g["v"], g["beta_k"], alpha=g["alpha"], beta_v=g["beta_v"], chunk=p.chunk,
                        o=sl["o"], S_T=sl["S"], workspace=ws_buf, stream=st)
        dr.dr_decode_step(gn["q"], gn["k"], gn["v"], gn["beta_k"], sl["S"], alpha=gn["alpha"], beta_v=gn["beta_v"],
                          o=sl["o1"], stream=st)
        sl["done"].record(st)
        s_out.wait_event(sl["done"])
        with torch.cuda.stream(s_out):
            sl["o_h"].copy_(sl["o"], non_blocking=True)
            sl["S_h"].copy_(sl["S"], non_blocking=True)
            sl["o1_h"].copy_(sl["o1"], non_blocking=True)
        sl["out"].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(ws)
    e0.record(st)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    st.wait_stream(s_in)
    st.wait_stream(s_out)
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), ws, dev) / e2e_steps
    # the last step's results, as read back, against the same step computed on the device alone
    last = slots[(e2e_steps - 1) % 2]
    if not (torch.equal(last["o_h"], o.cpu()) and torch.equal(last["o1_h"], o1.cpu())):
        raise RuntimeError("end-to-end results differ from the device-resident run")
    e2e = {"value": tok_heads * ws / (e2e_ms / 1e3) / 1e6, "unit": "Mtokens·heads/s", "ms_per_step": e2e_ms,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "pipeline": "2 slots; copies in, kernels and copies out on three streams"}
    del slots, host, host_n

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(p)

    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "Mtokens·heads/s", "n_gpus": ws, "steps": n,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": p.name, "B": p.B, "H": p.H, "T": p.T, "dk": p.dk, "dv": p.dv, "chunk": p.chunk,
                   "step": "chunkwise prefill of T tokens + one decode step per (b,h)", "parallelism": f"dp{ws}",
                   "l2": "inputs (2.4 GB per rank) larger than the 126 MB L2; no flush between steps",
                   "pipeline": ("step i's handoff decode on a second stream beside step i+1's prefill"
                                if pipelined else "serial: prefill, then its handoff decode, on one stream")},
        "prefill_ms": prefill_ms, "handoff_decode_ms": handoff_ms, "step_serial_ms": prefill_ms + handoff_ms,
        "roofline": roofline, "workloads": workloads, "decode": decode, "e2e": e2e, "cpu_baseline": cpu,
        "gpu_launches": 2 * n, "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
