"""GDPA benchmark: useful TFLOP/s of a forward + backward training step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-e2e] [--no-cpu-baseline]

One step is the whole hot path on one batch: the gated softmax training
workload (B=4096 samples, H=8, D=128, query lengths uniform in [256, 1024],
256 context-generated keys per sample, log-sigmoid gate, dO ~ N(0,1)) through
gdpa_forward then gdpa_backward.  Useful FLOPs count 4*D per visible
(query, key) pair and head in the forward and 8*D in the backward (padding and
recomputation excluded).  The inputs (about 15 GB) are larger than the 126 MB
L2, so no flush is needed between steps.

Multi-GPU (torchrun, one process per GPU): samples are independent, so each
rank runs its own full batch (weak scaling) with no collective on the data
path; the time is the max over ranks of the CUDA-event time.

--impl reference times the fp64 CPU oracle (the only other implementation
there is) on the host cores, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, make_workload  # noqa: E402

METRIC = "GDPA fwd/bwd useful TFLOP/s on 1 B200; % of dense BF16 tensor peak"
WORKLOADS = {CONFIGS[c]["name"]: c for c in CONFIGS}
DEFAULT_WORKLOAD = CONFIGS[5]["name"]
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- accounting
def visible_pairs_per_sample(w) -> np.ndarray:
    """Visible (query, key) pairs of each sample (per head)."""
    ql, kl = w.q_lens.astype(np.int64), w.kv_lens.astype(np.int64)
    if w.window_left < 0 and w.window_right < 0:
        return ql * kl
    out = np.zeros(w.B, np.int64)
    for b in range(w.B):
        i = np.arange(ql[b])
        lo = np.maximum(0, i - w.window_left) if w.window_left >= 0 else np.zeros_like(i)
        hi = (np.minimum(kl[b] - 1, i + w.window_right) if w.window_right >= 0
              else np.full_like(i, kl[b] - 1))
        out[b] = np.maximum(0, hi - lo + 1).sum()
    return out


def useful_flops(w, backward: bool) -> tuple[float, float]:
    pairs = float(visible_pairs_per_sample(w).sum()) * w.H
    fwd = 4.0 * w.D * pairs
    bwd = 8.0 * w.D * pairs if backward else 0.0
    return fwd, bwd


def algorithmic_bytes(w, backward: bool) -> tuple[float, float]:
    """Bytes a perfect kernel must move: each input read once, each output
    written once (bf16 tensors, fp32 gate/LSE)."""
    tq, tk, H, D = w.total_q, w.total_kv, w.H, w.D
    gate = 4.0 * H * tk if w.bias_kind else 0.0
    lse = 4.0 * H * tq if w.phi == 1 else 0.0
    fwd = 2.0 * H * D * (tq + 2 * tk + tq) + gate + lse           # Q, K, V -> O (+ LSE)
    bwd = 0.0
    if backward:
        bwd = (2.0 * H * D * (tq * 4 + tk * 4)                     # Q, O, dO, dQ; K, V, dK, dV
               + 2 * gate + lse)                                    # gate read, its gradient written
    return fwd, bwd


# per entry of profiles/traffic.json: the sources of the kernels whose DRAM
# bytes it records (the schedule kernel's few bytes are not in those figures)
KERNEL_SOURCES = {
    "gdpa_backward": ["gdpa_bwd.cu", "gdpa_internal.h", "sm100.cuh"],
    "gdpa_forward": ["gdpa_fwd.cu", "gdpa_internal.h", "sm100.cuh", "gdpa_pdl.cuh"],
    "gdpa_sumkron_forward": ["gdpa_sumkron.cu", "gdpa_ops.h", "gdpa_internal.h", "sm100.cuh"],
    "gdpa_rotary_apply": ["gdpa_rotary.cu", "gdpa_ops.h", "gdpa_internal.h", "sm100.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "pffn_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, n_samples: int):
    """DRAM bytes per launch from the committed ncu capture (profiles/
    traffic.json), scaled by samples; None when the kernel's sources changed
    since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("source_hash") != kernel_source_hash(kernel):
        return None
    return d["dram_bytes"] / d["samples"] * n_samples


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, \
            "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- ranks
def rank_seed(cfg: int, rank: int) -> int:
    """Each rank draws its own batch: independent samples, no shared data."""
    return cfg + 1000 * rank


def max_over_ranks(x: float, device) -> float:
    """The job's time is the slowest rank's (MAX all-reduce of one number)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's useful FLOPs over the slowest time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling during the timed region (clocks and throttle reasons)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="gdpa_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- our arm
def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from pffn_attention_b200 import gdpa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = WORKLOADS[args.workload]
    training = cfg == 5
    # each rank owns an independent batch of the same distribution
    w = make_workload(cfg, B=args.batch, device=dev, seed=rank_seed(cfg, rank),
                      with_dout=training, **phi_override(args))
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
    p = gdpa.make_params(w.B, w.H, w.D, w.total_q, w.total_kv, phi=w.phi, scale=w.scale,
                         window=(w.window_left, w.window_right), bias_kind=w.bias_kind,
                         max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv)
    o = torch.empty_like(w.q)
    lse = torch.empty((w.H, w.total_q), dtype=torch.float32, device=dev)
    ws_f = gdpa.workspace_for(p, False, dev)
    if training:
        dq, dk, dv = torch.empty_like(w.q), torch.empty_like(w.k), torch.empty_like(w.v)
        # a training step also needs the gate's gradient (the gate is an input
        # computed upstream)
        dbias = (torch.empty((w.H, w.total_kv), dtype=torch.float32, device=dev)
                 if w.bias is not None else None)
        ws_b = gdpa.workspace_for(p, True, dev)
    stream = torch.cuda.Stream(device=dev)
    sh = stream.cuda_stream
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rc = gdpa.gdpa_forward(p, ptr(w.q), ptr(w.k), ptr(w.v), ptr(qo), ptr(ko), ptr(w.bias),
                               ptr(o), ptr(lse), ptr(ws_f), ws_f.numel(), sh)
        if rc:
            raise gdpa.GdpaError(rc, "gdpa_forward")
        if ev is not None:
            ev[1].record(stream)
        if training:
            rc = gdpa.gdpa_backward(p, ptr(w.q), ptr(w.k), ptr(w.v), ptr(o), ptr(w.dout), ptr(lse),
                                    ptr(qo), ptr(ko), ptr(w.bias), ptr(dq), ptr(dk), ptr(dv),
                                    ptr(dbias), ptr(ws_b), ws_b.numel(), sh)
            if rc:
                raise gdpa.GdpaError(rc, "gdpa_backward")
        if ev is not None:
            ev[2].record(stream)

    launches_per_step = 2 + (3 if training else 0)  # schedule+fwd, schedule+delta+bwd
    torch.cuda.synchronize(dev)  # inputs were generated on the default stream
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    st = gdpa.gdpa_get_device_status(ptr(ws_f), sh)
    if st or (training and gdpa.gdpa_get_device_status(ptr(ws_b), sh)):
        raise RuntimeError(f"device status after warm-up: {st}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local_rank))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) if training else 0.0

    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps

    f_fwd, f_bwd = useful_flops(w, training)
    b_fwd, b_bwd = algorithmic_bytes(w, training)
    value = job_tflops(f_fwd + f_bwd, world, ms_per_step)
    peaks, peak_src = load_peaks()

    # dominant call: the backward in a training step, else the forward
    if training:
        dom_name, dom_ms, dom_bytes, dom_flops = "gdpa_backward", bwd_ms, b_bwd, f_bwd
    else:
        dom_name, dom_ms, dom_bytes, dom_flops = "gdpa_forward", fwd_ms, b_fwd, f_fwd
    achieved_gbs = dom_bytes / (dom_ms * 1e-3) / 1e9
    # the committed capture is of the default workload; other runs report none
    traffic = (measured_traffic(dom_name, w.B)
               if args.workload == DEFAULT_WORKLOAD and not args.phi else None)
    roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
                "spec_peak": SPEC_HBM_GBS, "spec_frac": round(achieved_gbs / SPEC_HBM_GBS, 4),
                "traffic": None if traffic is None else round(traffic / 1e9, 3),
                "traffic_unit": "GB per launch", "algorithmic": round(dom_bytes / 1e9, 3),
                "kernel": dom_name, "peak_source": peak_src,
                "tensor_tflops": round(dom_flops / (dom_ms * 1e-3) / 1e12, 1),
                "tensor_frac": round(dom_flops / (dom_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, p, qo, ko, training, dev, world)
    per_workload = None
    if world == 1 and args.workload == DEFAULT_WORKLOAD and args.batch is None \
            and not args.no_per_workload:
        per_workload = run_per_workload(args, dev, peaks, peak_src)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload + ("" if args.batch is None else
                                                f" (batch {args.batch}, profiling)"),
                   "B": w.B, "H": w.H, "D": w.D,
                   "global_batch": w.B * world, "seq_len": f"q U[256,1024] / kv 256"
                   if cfg == 5 else "see workload", "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (no flush)",
                   "phi": {v: k for k, v in PHI_NAMES.items()}[w.phi],
                   "gate_grad": bool(training and w.bias is not None)},
        "pct_of_peak": {"measured_burst": round(value / world / peaks["bf16_tflops"], 4),
                        "measured_sustained": round(value / world
                                                    / peaks["bf16_tflops_sustained"], 4),
                        "spec": round(value / world / SPEC_BF16_TFLOPS, 4)},
        "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
        "fwd_tflops": round(f_fwd / (fwd_ms * 1e-3) / 1e12, 1),
        "bwd_tflops": round(f_bwd / (bwd_ms * 1e-3) / 1e12, 1) if training else None,
        "roofline": roofline,
        "per_workload": per_workload,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
    }
    return line, w


def run_per_workload(args, dev, peaks, peak_src):
    """The three forward-only workloads at full size (PFFN SiLU, seed pooling,
    sliding window): each timed as its own gdpa_forward call after 5 warm-ups,
    as the mean of 20 calls back to back between two CUDA events (and, beside
    it, the median of 20 calls each between its own events), inputs (0.6 to
    6 GB) larger than L2.  Useful TFLOP/s, and algorithmic bytes over time as a fraction of the
    measured HBM copy bandwidth and of the 8 TB/s spec."""
    import torch

    from pffn_attention_b200 import gdpa
    out = {}
    stream = torch.cuda.Stream(device=dev)
    for cfg in (2, 3, 4):
        w = make_workload(cfg, device=dev, seed=cfg, with_dout=False)
        qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
        ko = torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev)
        kw = dict(phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right),
                  bias=w.bias, bias_kind=w.bias_kind, max_seqlen_q=w.max_q,
                  max_seqlen_kv=w.max_kv, stream=stream)
        torch.cuda.synchronize(dev)
        o, lse, ws = gdpa.forward(w.q, w.k, w.v, qo, ko, **kw)
        for _ in range(5):
            gdpa.forward(w.q, w.k, w.v, qo, ko, out=o, lse=lse, workspace=ws, **kw)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(20)]
        for e0, e1 in evs:
            e0.record(stream)
            gdpa.forward(w.q, w.k, w.v, qo, ko, out=o, lse=lse, workspace=ws, **kw)
            e1.record(stream)
        # the same calls back to back between one pair of events: the device
        # time per call of a stream of calls, without the host's per-call
        # enqueue time showing up between a call's events
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(20):
            gdpa.forward(w.q, w.k, w.v, qo, ko, out=o, lse=lse, workspace=ws, **kw)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        if gdpa.device_status(ws, stream) != 0:
            raise RuntimeError(f"device status after {w.name}")
        single_ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
        ms = t0.elapsed_time(t1) / 20
        fl, _ = useful_flops(w, False)
        by, _ = algorithmic_bytes(w, False)
        gbs = by / (ms * 1e-3) / 1e9
        tf = fl / (ms * 1e-3) / 1e12
        out[w.name] = {"B": w.B, "H": w.H, "D": w.D, "fwd_ms": round(ms, 4),
                       "single_call_ms": round(single_ms, 4),
                       "useful_tflops": round(tf, 1),
                       "tensor_frac": round(tf / peaks["bf16_tflops"], 4),
                       "algorithmic_gb": round(by / 1e9, 3), "achieved_gbs": round(gbs, 1),
                       "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                       "hbm_frac_spec": round(gbs / SPEC_HBM_GBS, 4), "bound": "hbm",
                       "peak_source": peak_src,
                       "timing": "fwd_ms: mean of 20 back-to-back calls; single_call_ms: "
                                 "median of 20 calls each between its own events; 5 warm-ups"}
        del w, o, lse, ws, qo, ko
        torch.cuda.empty_cache()
    return out


def run_e2e(args, w, p, qo, ko, training, dev, world):
    """Same metric through the C ABI with host buffers: every step copies the
    inputs from pinned host memory and reads all outputs back.  Steps are
    pipelined the way a training loop feeds a GPU: step i + 1's host-to-device
    copies (one stream) run while step i's outputs go back to the host (another
    stream); a step's kernels wait for their own inputs and for the previous
    step's outputs to have been read back, and a step's input copies wait for
    the previous step's kernels.  If that path raises, or its last read-back
    does not hold the device's output, the steps run one after another on one
    stream instead, and the line says so."""
    import torch

    from pffn_attention_b200 import gdpa

    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    names = ["q", "k", "v"] + (["bias"] if w.bias is not None else []) + \
        (["dout"] if training else [])
    host_in = {n: pinned_copy(getattr(w, n)) for n in names}
    host_qo = qo.cpu().pin_memory()
    host_ko = ko.cpu().pin_memory()
    dev_in = {n: torch.empty_like(t, device=dev) for n, t in host_in.items()}
    dqo, dko = torch.empty_like(qo), torch.empty_like(ko)
    o = torch.empty_like(dev_in["q"])
    lse = torch.empty((w.H, w.total_q), dtype=torch.float32, device=dev)
    outs = {"o": o}
    if training:
        outs.update(dq=torch.empty_like(dev_in["q"]), dk=torch.empty_like(dev_in["k"]),
                    dv=torch.empty_like(dev_in["v"]))
        if w.bias is not None:
            outs["dbias"] = torch.empty((w.H, w.total_kv), dtype=torch.float32, device=dev)
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in outs.items()}
    ws_f = gdpa.workspace_for(p, False, dev)
    ws_b = gdpa.workspace_for(p, True, dev) if training else None
    stream = torch.cuda.Stream(device=dev)   # the kernels
    cin = torch.cuda.Stream(device=dev)      # host-to-device copies
    cout = torch.cuda.Stream(device=dev)     # device-to-host copies
    sh = stream.cuda_stream
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + \
        host_qo.numel() * 4 + host_ko.numel() * 4
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())

    def copy_in(s):
        with torch.cuda.stream(s):
            for n, t in host_in.items():
                dev_in[n].copy_(t, non_blocking=True)
            dqo.copy_(host_qo, non_blocking=True)
            dko.copy_(host_ko, non_blocking=True)

    def compute():
        rc = gdpa.gdpa_forward(p, ptr(dev_in["q"]), ptr(dev_in["k"]), ptr(dev_in["v"]), ptr(dqo),
                               ptr(dko), ptr(dev_in.get("bias")), ptr(o), ptr(lse), ptr(ws_f),
                               ws_f.numel(), sh)
        assert rc == 0, rc
        if training:
            rc = gdpa.gdpa_backward(p, ptr(dev_in["q"]), ptr(dev_in["k"]), ptr(dev_in["v"]), ptr(o),
                                    ptr(dev_in["dout"]), ptr(lse), ptr(dqo), ptr(dko),
                                    ptr(dev_in.get("bias")), ptr(outs["dq"]), ptr(outs["dk"]),
                                    ptr(outs["dv"]), ptr(outs.get("dbias")), ptr(ws_b),
                                    ws_b.numel(), sh)
            assert rc == 0, rc

    def copy_out(s):
        with torch.cuda.stream(s):
            for n, t in outs.items():
                host_out[n].copy_(t, non_blocking=True)

    def step_sequential():
        copy_in(stream)
        compute()
        copy_out(stream)

    in_ready, comp_done, out_read = (torch.cuda.Event() for _ in range(3))

    def step_pipelined():
        cin.wait_event(comp_done)     # the previous step's kernels have read the inputs
        copy_in(cin)
        in_ready.record(cin)
        stream.wait_event(in_ready)
        stream.wait_event(out_read)   # the previous step's outputs are back on the host
        compute()
        comp_done.record(stream)
        cout.wait_event(comp_done)
        copy_out(cout)
        out_read.record(cout)

    steps = max(2, min(args.steps, 5))

    n_chk = min(4096, o.shape[0])

    def timed(step_fn, first, last):
        for _ in range(2):
            step_fn()
        torch.cuda.synchronize(dev)
        # rows the check below reads: cleared on the host, so only a read-back
        # made inside the timed steps can fill them
        host_out["o"][:n_chk].zero_()
        host_out["o"][-n_chk:].zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(first)
        for _ in range(steps):
            step_fn()
        e1.record(last)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    mode, note = "pipelined", None
    try:
        ms = timed(step_pipelined, cin, cout)
        # the last read-back holds what the kernels wrote (rows at both ends)
        ok = (torch.equal(host_out["o"][:n_chk], o[:n_chk].cpu())
              and torch.equal(host_out["o"][-n_chk:], o[-n_chk:].cpu()))
        if not ok:
            raise RuntimeError("read-back does not match the device output")
    except Exception as e:  # noqa: BLE001 -- fall back to the one-stream steps
        torch.cuda.synchronize(dev)
        mode, note = "sequential", f"pipelined steps failed: {e}"[:200]
        ms = timed(step_sequential, stream, stream)
    ms = max_over_ranks(ms, dev)
    f_fwd, f_bwd = useful_flops(w, training)
    line = {"value": round(job_tflops(f_fwd + f_bwd, world, ms), 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "steps": steps, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "mode": mode}
    if note:
        line["note"] = note
    return line


# ----------------------------------------------------------------- the oracle
def oracle_sample(cfg: int, n_samples: int, seed: int, training: bool, **kw):
    """A fresh batch of n_samples drawn from the workload's distributions."""
    return make_workload(cfg, B=n_samples, seed=seed, device="cpu", with_dout=training, **kw)


PHI_NAMES = {"silu": 0, "softmax": 1, "identity": 2, "gelu": 3}


def phi_override(args) -> dict:
    """--phi replaces the workload's activation (diagnostic runs)."""
    return {"phi": PHI_NAMES[args.phi]} if getattr(args, "phi", None) else {}


def time_oracle(sub, training: bool) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.forward_workload(sub)
    if training:
        oracle.backward_workload(sub)
    return time.perf_counter() - t0


def cpu_baseline(args, w, training: bool, target_s: float = 16.0) -> dict:
    """The fp64 oracle, as it stands, on a bounded sample of the same workload."""
    import oracle
    cfg = WORKLOADS[args.workload]
    n = 2
    dt = time_oracle(oracle_sample(cfg, n, 7000, training, **phi_override(args)), training)
    n = int(min(w.B, max(2, n * target_s / max(dt, 1e-3))))
    sub = oracle_sample(cfg, n, 7001, training, **phi_override(args))
    dt = time_oracle(sub, training)
    f_fwd, f_bwd = useful_flops(sub, training)
    return {"value": round((f_fwd + f_bwd) / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} samples drawn from {args.workload}'s distributions (all {sub.H} "
                      f"heads, {int(sub.total_q)} query rows), fwd{'+bwd' if training else ''}, "
                      f"{dt:.1f} s"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    import oracle
    cfg = WORKLOADS[args.workload]
    training = cfg == 5
    per_step = 6 if training else 64
    for i in range(args.warmup):
        time_oracle(oracle_sample(cfg, 2, 100 + i, training, **phi_override(args)), training)
    times, flops = [], 0.0
    for i in range(args.steps):
        sub = oracle_sample(cfg, per_step, 200 + i, training, **phi_override(args))
        times.append(time_oracle(sub, training))
        f, b = useful_flops(sub, training)
        flops += f + b
    total = sum(times)
    value = flops / total / 1e12
    sample = (f"{per_step} samples per step drawn from {args.workload}'s distributions "
              f"(all heads)")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                             "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------- main
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------- grouped
# Event-level personalisation: each event type runs its own small GDPA problem
# with its own heads, width, activation and window.  A synthetic set of eight
# event types (shapes chosen across the workloads' ranges) timed as one
# gdpa_forward_grouped call against the same problems as separate calls.
EVENT_TYPES = [  # (H, D, phi, window, B, q lengths, kv lengths ("same" = q), bias)
    (8, 128, 1, (255, 0), 64, (200, 1000), "same", 0),
    (4, 128, 1, (127, 0), 128, (100, 500), "same", 0),
    (4, 64, 1, (63, 0), 256, (50, 300), "same", 0),
    (2, 64, 0, (-1, -1), 512, (20, 200), (64, 64), 0),
    (2, 32, 1, (31, 0), 512, (10, 100), "same", 0),
    (8, 128, 1, (-1, -1), 128, (100, 600), (256, 256), 2),
    (4, 64, 3, (-1, -1), 256, (50, 400), (64, 64), 0),
    (2, 32, 0, (-1, -1), 1024, (1, 64), (16, 16), 0),
]


def run_grouped(args):
    import torch

    from pffn_attention_b200 import gdpa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    names = {v: k for k, v in PHI_NAMES.items()}
    rng = np.random.default_rng(600)
    ws_, probs, flops, byts = [], [], 0.0, 0.0
    for i, (H, D, phi, win, B, ql, kl, bias) in enumerate(EVENT_TYPES):
        q_lens = rng.integers(ql[0], ql[1] + 1, B)
        kv_lens = q_lens if kl == "same" else rng.integers(kl[0], kl[1] + 1, B)
        base = 3 if phi == 1 else 2
        extra = {} if phi == 1 else dict(scale=1.0, kv_std=1.0 / np.sqrt(D))
        w = make_workload(base, seed=610 + i, q_lens=q_lens, kv_lens=kv_lens, H=H, D=D, phi=phi,
                          window=win, bias=bias, device=dev, with_dout=False, **extra)
        ws_.append(w)
        probs.append(dict(q=w.q, k=w.k, v=w.v,
                          q_offsets=torch.tensor(w.q_offsets, dtype=torch.int32, device=dev),
                          kv_offsets=torch.tensor(w.kv_offsets, dtype=torch.int32, device=dev),
                          bias=w.bias, phi=names[phi], scale=w.scale, window=win,
                          bias_kind=bias, max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv))
        flops += useful_flops(w, False)[0]
        byts += algorithmic_bytes(w, False)[0]
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    outs, wsg = gdpa.forward_grouped(probs, stream=stream)  # allocates outputs, workspace
    single = []
    for d, (o, lse) in zip(probs, outs):
        kw = {k: d[k] for k in ("phi", "scale", "window", "bias", "bias_kind", "max_seqlen_q",
                                "max_seqlen_kv")}
        _, _, ws1 = gdpa.forward(d["q"], d["k"], d["v"], d["q_offsets"], d["kv_offsets"], out=o,
                                 lse=lse, stream=stream, **kw)  # its workspace, reused below
        single.append((d, kw, o, lse, ws1))

    def grouped_step():
        gdpa.forward_grouped(probs, workspace=wsg, stream=stream)

    def separate_step():
        for d, kw, o, lse, ws1 in single:
            gdpa.forward(d["q"], d["k"], d["v"], d["q_offsets"], d["kv_offsets"], out=o,
                         lse=lse, workspace=ws1, stream=stream, **kw)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    g_ms = timed(grouped_step)
    s_ms = timed(separate_step)
    assert gdpa.device_status(wsg, stream) == 0
    return {"metric": "GDPA grouped forward, event-type problems per call (useful TFLOP/s)",
            "value": round(flops / (g_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(g_ms, 4),
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "event_groups", "problems": len(EVENT_TYPES),
                       "samples": int(sum(w.B for w in ws_))},
            "separate_calls_ms": round(s_ms, 4), "grouped_speedup": round(s_ms / g_ms, 3),
            "achieved_gbs": round(byts / (g_ms * 1e-3) / 1e9, 1)}


def run_rotary(args):
    """Forward of the sliding-window self-attention workload with the rotary
    temporal embedding (Q and K turned in shared memory) against the same
    forward without it; the table build is timed on its own."""
    import torch

    from pffn_attention_b200 import gdpa
    from workloads import EVENT_TIME_SCALE, event_times
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = make_workload(4, device=dev, with_dout=True)
    stream = torch.cuda.Stream(device=dev)
    qo = torch.tensor(w.q_offsets, dtype=torch.int32, device=dev)
    times = torch.tensor(event_times(w.q_lens, 4), dtype=torch.int64, device=dev)
    kw = dict(phi=w.phi, scale=w.scale, window=(w.window_left, w.window_right),
              max_seqlen_q=w.max_q, max_seqlen_kv=w.max_kv, stream=stream)
    table = gdpa.rotary_table(qo, times, w.D, EVENT_TIME_SCALE, stream=stream)
    o, lse, ws = gdpa.forward(w.q, w.k, w.v, qo, qo, rope=(table, table), **kw)
    o2, lse2, ws2 = gdpa.forward(w.q, w.k, w.v, qo, qo, **kw)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    r_ms = timed(lambda: gdpa.forward(w.q, w.k, w.v, qo, qo, rope=(table, table), out=o, lse=lse,
                                      workspace=ws, **kw))
    p_ms = timed(lambda: gdpa.forward(w.q, w.k, w.v, qo, qo, out=o2, lse=lse2, workspace=ws2,
                                      **kw))
    t_ms = timed(lambda: gdpa.rotary_table(qo, times, w.D, EVENT_TIME_SCALE, out=table,
                                           stream=stream))
    qr, kr = torch.empty_like(w.q), torch.empty_like(w.k)
    a_ms = timed(lambda: (gdpa.rotary_apply(w.q, table, out=qr, stream=stream),
                          gdpa.rotary_apply(w.k, table, out=kr, stream=stream)))
    # training step (forward + backward), with and without the rotary turn
    dq, dk, dv = torch.empty_like(w.q), torch.empty_like(w.k), torch.empty_like(w.v)
    _, _, _, wsb = gdpa.backward(w.q, w.k, w.v, o, w.dout, lse, qo, qo, rope=(table, table),
                                 dq=dq, dk=dk, dv=dv, **kw)
    _, _, _, wsb2 = gdpa.backward(w.q, w.k, w.v, o2, w.dout, lse2, qo, qo, dq=dq, dk=dk, dv=dv,
                                  **kw)

    def step(rope):
        if rope:
            gdpa.forward(w.q, w.k, w.v, qo, qo, rope=(table, table), out=o, lse=lse, workspace=ws,
                         **kw)
            gdpa.backward(w.q, w.k, w.v, o, w.dout, lse, qo, qo, rope=(table, table), dq=dq,
                          dk=dk, dv=dv, workspace=wsb, **kw)
        else:
            gdpa.forward(w.q, w.k, w.v, qo, qo, out=o2, lse=lse2, workspace=ws2, **kw)
            gdpa.backward(w.q, w.k, w.v, o2, w.dout, lse2, qo, qo, dq=dq, dk=dk, dv=dv,
                          workspace=wsb2, **kw)
    sr_ms = timed(lambda: step(True))
    sp_ms = timed(lambda: step(False))

    # the same training step composed from the exported turn: Q and K turned
    # once for both calls, dQ and dK turned back at the end (two passes)
    def composed():
        gdpa.rotary_apply(w.q, table, out=qr, stream=stream)
        gdpa.rotary_apply(w.k, table, out=kr, stream=stream)
        gdpa.forward(qr, kr, w.v, qo, qo, out=o2, lse=lse2, workspace=ws2, **kw)
        gdpa.backward(qr, kr, w.v, o2, w.dout, lse2, qo, qo, dq=dq, dk=dk, dv=dv,
                      workspace=wsb2, **kw)
        gdpa.rotary_apply(dq, table, inverse=True, out=dq, stream=stream)
        gdpa.rotary_apply(dk, table, inverse=True, out=dk, stream=stream)
    sc_ms = timed(composed)
    assert gdpa.device_status(wsb, stream) == 0
    assert gdpa.device_status(ws, stream) == 0
    flops = useful_flops(w, False)[0]
    byts = algorithmic_bytes(w, False)[0] + table.numel() * 4  # + one read of the table
    turn_bytes = 2.0 * 2 * (w.q.numel() + w.k.numel()) + 2.0 * table.numel() * 4
    peaks, src = load_peaks()
    return {"metric": "GDPA forward with rotary temporal embedding, sliding-window "
                      "self-attention (useful TFLOP/s)",
            "value": round(flops / (r_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r_ms, 4),
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "D": w.D,
                       "window": [w.window_left, w.window_right], "l2": "inputs > L2"},
            "plain_forward_ms": round(p_ms, 4), "rotary_overhead": round(r_ms / p_ms, 3),
            "table_ms": round(t_ms, 4), "achieved_gbs": round(byts / (r_ms * 1e-3) / 1e9, 1),
            "train_step_ms": round(sr_ms, 4), "plain_train_step_ms": round(sp_ms, 4),
            "train_rotary_overhead": round(sr_ms / sp_ms, 3),
            "train_step_composed_ms": round(sc_ms, 4),
            # the turn pass (Q and K read and written, the table read once per tensor)
            "roofline": {"bound": "hbm", "kernel": "gdpa_rotary_apply", "ms": round(a_ms, 4),
                         "achieved": round(turn_bytes / (a_ms * 1e-3) / 1e9, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(turn_bytes / (a_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                         "traffic": measured_traffic("gdpa_rotary_apply", w.B),
                         "algorithmic": turn_bytes, "peak_source": src}}


def run_sumkron(args):
    """SumKronLinear forward and backward on the page's typical configuration
    (seed summaries of the seed-pooling batch).  Useful FLOPs of the cheaper
    association: forward 2 k T S D + 2 k T D^2 per sample; backward twice
    that (dY W^T, A^T U, U X^T, Z^T dY; the recomputed Z = A X excluded)."""
    import torch

    from pffn_attention_b200 import gdpa
    from workloads import SUMKRON_CONFIG, make_sumkron
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    c = SUMKRON_CONFIG
    B, S, T, D, k = c["B"], c["S"], c["T"], c["D"], c["k"]
    x, a, w = make_sumkron(B, S, T, D, k, seed=1, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(2)
    dy = torch.randn((B, T, D), generator=gen, device=dev).to(torch.bfloat16)
    stream = torch.cuda.Stream(device=dev)
    y, ws = gdpa.sumkron_forward(x, a, w, stream=stream)
    _, _, _, wsb = gdpa.sumkron_backward(x, a, w, dy, stream=stream)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    ms_f = timed(lambda: gdpa.sumkron_forward(x, a, w, out=y, workspace=ws, stream=stream))
    assert gdpa.device_status(ws, stream) == 0
    ms_b = timed(lambda: gdpa.sumkron_backward(x, a, w, dy, workspace=wsb, stream=stream))
    assert gdpa.device_status(wsb, stream) == 0
    flops_f = B * (2.0 * k * T * S * D + 2.0 * k * T * D * D)
    flops_b = 2.0 * flops_f
    byts = 2.0 * (x.numel() + y.numel() + a.numel() + w.numel())
    peaks, src = load_peaks()
    tf_f = flops_f / (ms_f * 1e-3) / 1e12
    tf_b = flops_b / (ms_b * 1e-3) / 1e12
    tf = (flops_f + flops_b) / ((ms_f + ms_b) * 1e-3) / 1e12
    return {"metric": "SumKronLinear forward + backward, HSP second stage (useful TFLOP/s)",
            "value": round(tf, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_f + ms_b, 4),
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "sumkron_hsp", **c, "l2": "inputs > L2"},
            "fwd_ms": round(ms_f, 4), "fwd_tflops": round(tf_f, 2),
            "bwd_ms": round(ms_b, 4), "bwd_tflops": round(tf_b, 2),
            "roofline": {"bound": "tensor", "achieved": round(tf_f, 2),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf_f / peaks["bf16_tflops"], 4),
                         "kernel": "gdpa_sumkron_forward",
                         "traffic": measured_traffic("gdpa_sumkron_forward", B),
                         "traffic_unit": "bytes per launch", "algorithmic": byts,
                         "peak_source": src,
                         "bwd_frac": round(tf_b / peaks["bf16_tflops"], 4)},
            "achieved_gbs": round(byts / (ms_f * 1e-3) / 1e9, 1)}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=None,
                    help="samples per rank (default: the workload's full batch); smaller "
                         "batches are for profiling captures")
    ap.add_argument("--phi", choices=sorted(PHI_NAMES), default=None,
                    help="replace the workload's activation (diagnostics)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the forward-only workloads' per-workload timings")
    ap.add_argument("--grouped", action="store_true",
                    help="time the event-type problems as one grouped call vs separate calls")
    ap.add_argument("--rotary", action="store_true",
                    help="time the sliding-window forward with the rotary temporal embedding")
    ap.add_argument("--sumkron", action="store_true",
                    help="time the SumKronLinear forward and backward (HSP second stage)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    rank, world, local = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.grouped:
        if world != 1 or args.impl != "ours":
            ap.error("--grouped runs on one GPU, our implementation")
        print(json.dumps(run_grouped(args)), flush=True)
        return 0
    if args.sumkron:
        if world != 1 or args.impl != "ours":
            ap.error("--sumkron runs on one GPU, our implementation")
        print(json.dumps(run_sumkron(args)), flush=True)
        return 0
    if args.rotary:
        if world != 1 or args.impl != "ours":
            ap.error("--rotary runs on one GPU, our implementation")
        print(json.dumps(run_rotary(args)), flush=True)
        return 0

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        line, w = run_ours(args, rank, world, local)
        if rank == 0:
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(args, w, WORKLOADS[args.workload] == 5)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
