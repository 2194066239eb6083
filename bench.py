#!/usr/bin/env python
"""Benchmark of the gated delta-rule chunked forward on B200.

Prints ONE JSON line on rank 0.  Default workload: the Gated DeltaNet layer
forward at 350M-model shape (B=8, T=4096, H=16, d_k=d_v=128, C=64, bf16
q/k/v, fp32 gates and state, S0 = 0, S_T returned).  A "step" is one
gdr_chunk_fwd call over that batch.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle, bounded sample

Multi-GPU (launched by torchrun): every rank runs the same per-GPU workload
on its own seeded batch (independent (b, h) problems, no collective on the
data path) -> weak scaling; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from gated_delta_rule_93_b200.inputs import WORKLOADS, make_workload_inputs  # noqa: E402
from gated_delta_rule_93_b200.sharding import max_over_ranks  # noqa: E402

METRIC = "tokens/s and TFLOP/s per gated-delta layer fwd (1 B200), % of roofline"
DEFAULT_WORKLOAD = "gdn_b8_t4096_h16_d128"
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCES = {
    # the kernel each kind of workload times, for the profile's source hash
    "chunk": ["gated_delta_rule_93_b200/csrc/gdr_chunk_tc.cu",
              "gated_delta_rule_93_b200/csrc/gdr_sm100.cuh"],
    "seg": ["gated_delta_rule_93_b200/csrc/gdr_chunk_tc.cu",
            "gated_delta_rule_93_b200/csrc/gdr_segments.cu",
            "gated_delta_rule_93_b200/csrc/gdr_sm100.cuh"],
    "split": ["gated_delta_rule_93_b200/csrc/gdr_chunk_split.cu",
              "gated_delta_rule_93_b200/csrc/gdr_tc_util.cuh",
              "gated_delta_rule_93_b200/csrc/gdr_sm100.cuh"],
    "step": ["gated_delta_rule_93_b200/csrc/gdr_step.cu"],
    "bwd": ["gated_delta_rule_93_b200/csrc/gdr_bwd_tc.cu",
            "gated_delta_rule_93_b200/csrc/gdr_tc_util.cuh",
            "gated_delta_rule_93_b200/csrc/gdr_chunk_tc.cu",
            "gated_delta_rule_93_b200/csrc/gdr_sm100.cuh"],
    "dplr": ["gated_delta_rule_93_b200/csrc/gdr_chunk_split.cu",
             "gated_delta_rule_93_b200/csrc/gdr_tc_util.cuh",
             "gated_delta_rule_93_b200/csrc/gdr_sm100.cuh"],
}


def kernel_kind(w, launches=1):
    """Which kernel a workload times: the KERNEL_SOURCES key."""
    if w.backward:
        return "bwd"
    if w.mixer == "dplr":
        return "dplr"
    if w.kind == "step":
        return "step"
    if w.dtype != torch.bfloat16 or w.dk != 128 or w.dv != 128:
        return "split"
    return "seg" if launches > 1 else "chunk"


# ------------------------------------------------------------------ work model
def algorithmic_bytes(w):
    """HBM bytes a perfect fused kernel must move for one step (per GPU)."""
    e_in = 2 if w.dtype == torch.bfloat16 else 4
    gate_elems = w.dk if w.gate == "channel" else 1
    if w.kind == "step":  # one decode step: S read + written once, q/k/v/g/beta in, o out
        return w.B * w.H * (8 * w.dk * w.dv + (2 * w.dk + w.dv) * e_in + w.dv * e_in
                            + 4 * gate_elems + 4)
    beta = 0 if w.mixer == "gla" else 4
    per_tok = (2 * w.dk + w.dv) * e_in + w.dv * e_in + 4 * gate_elems + beta
    if w.mixer == "dplr":  # q, k, a, b, v, g in; o out
        per_tok = (4 * w.dk + w.dv) * e_in + w.dv * e_in + 4 * gate_elems
    if w.backward:  # q, k, v, g, beta, dL/do in; dq, dk, dv, dg, dbeta out (fp32)
        per_tok = ((2 * w.dk + w.dv) * e_in + 4 * gate_elems + 4 + 4 * w.dv
                   + 4 * (2 * w.dk + w.dv) + 4 * gate_elems + 4)
    state = 4 * w.dk * w.dv * w.B * w.H
    return w.B * w.T * w.H * per_tok + state * (int(w.with_S0) + int(w.want_S_T))


def algorithmic_flops(w, C=64):
    """Chunked-method flops per step, counting masked products as triangles:
    6 d_k d_v + C (3 d_k + 2 d_v) + C^2 / 3 per token-head (decode step:
    about 7 d_k d_v per state, CUDA cores)."""
    if w.kind == "step":
        return w.B * w.H * 7.0 * w.dk * w.dv
    if w.backward:  # one recomputed forward step (5 d^2) and its reverse (16 d^2)
        return w.B * w.T * w.H * 21.0 * w.dk * w.dv
    if w.mixer == "dplr":  # chunked: two state reads and two state updates (8 d_k d_v),
        # four masked intra-chunk products, three masked products with values
        per = 8 * w.dk * w.dv + C * (4 * w.dk + 3 * w.dv) + C * C / 3.0
        return w.B * w.T * w.H * per
    if w.mixer == "gla":  # no correction: state update, S q, masked Q K^T and P V
        return w.B * w.T * w.H * (4 * w.dk * w.dv + C * (w.dk + w.dv))
    per = 6 * w.dk * w.dv + C * (3 * w.dk + 2 * w.dv) + C * C / 3.0
    return w.B * w.T * w.H * per


def backward_on_tensor_cores(w):
    """The backward's tensor-core path: bf16, d_k = d_v = 128, scalar gate."""
    return (w.backward and w.dtype == torch.bfloat16 and w.dk == 128 and w.dv == 128
            and w.gate == "scalar" and w.T > 0)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_source_hash(kind="chunk"):
    """Hash of the sources of the kernel a workload times (profiles record it)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        p = os.path.join(ROOT, rel)
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kind="chunk"):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_source_hash(kind)
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == workload:
                if parts[2] == cur:
                    return float(parts[1])
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        # the first sample before the timed region starts (bounded)
        t_end = time.time() + 5.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        # one more sample after the timed region (a short region can fall
        # between two samples), bounded
        n0, t_end = len(self.lines), time.time() + 1.0
        while len(self.lines) <= n0 and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.005)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm
def make_step(w, dev, rank, nsteps):
    """The workload's inputs on the device and one step of it through the
    binding.  Returns a dict: step (callable), host (CPU inputs), d (device
    inputs), o, S_T, S (decode state), grads, results (what a step returns to
    its caller), launches (kernels per step)."""
    from gated_delta_rule_93_b200 import binding

    r = {"grads": None, "S": None, "S_T": None}
    if w.kind == "step":
        # decode: one gdr_step over all N x H states per step, inputs of the
        # first nsteps steps resident, the state updated in place
        host = make_workload_inputs(w, seed=rank, steps=nsteps)
        d = {k: v.to(dev) for k, v in host.items()}
        S = d["S0"].clone()
        o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=dev)
        it = [0]

        def step():
            i = it[0] % nsteps
            it[0] += 1
            binding.step(d["q"][i], d["k"][i], d["v"][i], d["g"][i], d["beta"][i], S, o=o)

        r.update(step=step, host=host, d=d, o=o, S=S, launches=1, results=[o])
        return r
    host = make_workload_inputs(w, seed=rank)
    d = {k: (v.to(dev) if v is not None else None) for k, v in host.items()}
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=w.dtype, device=dev)
    S_T = torch.empty(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=dev) \
        if w.want_S_T else None
    # scratch of the segment path (long sequences with few heads), if any
    ws_bytes = binding.chunk_fwd_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.C, w.dtype,
                                                 w.gate)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None
    launches = binding.chunk_fwd_kernel_launches(w.B, w.T, w.H, w.dk, w.dv, w.C, w.dtype,
                                                 w.gate)

    def step():
        binding.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o=o,
                          S_T=S_T, output_final_state=S_T is not None, workspace=ws)

    if w.prologue:  # raw projections in: one launch, no workspace
        launches = 1

        def step():
            binding.chunk_fwd_prologue(d["q"], d["k"], d["v"], d["a"], d["b"],
                                       d["gate_scale"], d["S0"], o=o, S_T=S_T,
                                       output_final_state=S_T is not None)

    grads = None
    if w.backward:  # gradients for a seeded dL/do; preallocated outputs and workspace
        # (tensor cores: the forward rerun with a stash, the reverse state
        # pass and the chunk-parallel gradient pass; else one CUDA-core launch)
        launches = 3 if backward_on_tensor_cores(w) else 1
        f32 = dict(dtype=torch.float32, device=dev)
        grads = dict(dq=torch.empty(w.B, w.T, w.H, w.dk, **f32),
                     dk=torch.empty(w.B, w.T, w.H, w.dk, **f32),
                     dv=torch.empty(w.B, w.T, w.H, w.dv, **f32),
                     dg=torch.empty(tuple(d["g"].shape), **f32),
                     dbeta=torch.empty(w.B, w.T, w.H, **f32), dS0=None)
        bws = torch.empty(binding.chunk_bwd_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.dtype,
                                                            w.gate),
                          dtype=torch.uint8, device=dev)
        o, S_T = grads["dq"], None

        def step():
            binding.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dout"], d["S0"],
                              None, want_dS0=False, workspace=bws, out=grads)

    if w.mixer == "dplr":  # chunked DPLR forward on the tensor cores: one launch
        launches = 1

        def step():
            binding.dplr_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["g"], d["S0"], o=o,
                             S_T=S_T, output_final_state=S_T is not None)

    if w.mixer == "gla":  # gated linear attention: one launch, no beta, no workspace
        host.pop("beta")
        d.pop("beta")
        launches = 1

        def step():
            binding.chunk_fwd_gla(d["q"], d["k"], d["v"], d["g"], d["S0"], o=o, S_T=S_T,
                                  output_final_state=S_T is not None)

    results = [grads[n] for n in ("dq", "dk", "dv", "dg", "dbeta")] if w.backward else \
        [o] + ([S_T] if S_T is not None else [])
    r.update(step=step, host=host, d=d, o=o, S_T=S_T, grads=grads, launches=launches,
             results=results)
    return r


def time_device(step, steps, warmup, dev, world, local_rank):
    """W untimed steps, then K steps timed with CUDA events on the launching
    stream between barriers and synchronisations, SM clocks sampled during
    the region.  Returns (total ms, per-step ms list, clocks)."""
    from gated_delta_rule_93_b200 import binding

    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    if binding.device_status() != 0:
        raise RuntimeError("device status word set during warm-up")
    vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    clocks = ClockSampler(vis[local_rank].strip() if local_rank < len(vis) else local_rank)
    clocks.start()
    time.sleep(0.15)
    barrier()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    # Hold the stream with a short spin (torch's, before the timed region)
    # while the host enqueues the K steps, so that the events time the
    # device's back-to-back execution and not the host's per-call latency
    # (which would dominate small workloads).
    torch.cuda._sleep(int(1e6 * (steps + 2)))
    t0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    if binding.device_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    return t0.elapsed_time(t1), [a.elapsed_time(b) for a, b in ev], clk


def roofline_fields(w, total_ms, per_launch_ms, steps, world, clk, launches=1):
    """tokens/s, TFLOP/s and the roofline of one timed workload."""
    ms_step = total_ms / steps
    tokens_step = w.B * w.T if w.kind == "chunk" else w.B  # tokens one step processes
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    abytes = algorithmic_bytes(w)
    aflops = algorithmic_flops(w, w.C)
    avg_launch_ms = sum(per_launch_ms) / len(per_launch_ms)
    achieved = abytes / (avg_launch_ms / 1e3) / 1e9
    roof_ms = max(abytes / (hbm_peak * 1e9), aflops / (tc_peak * 1e12)) * 1e3
    alu = w.backward and not backward_on_tensor_cores(w)
    alu_peak = None
    if alu:  # fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 flop x SM clock
        alu_peak = 148 * 128 * 2 * ((clk or {}).get("sm_max_mhz") or 1965.0) * 1e6 / 1e12
        roof_ms = max(abytes / (hbm_peak * 1e9), aflops / (alu_peak * 1e12)) * 1e3
    if alu:
        roof = {"bound": "alu", "achieved": aflops / (avg_launch_ms / 1e3) / 1e12,
                "peak": alu_peak, "unit": "TFLOP/s",
                "frac": aflops / (avg_launch_ms / 1e3) / 1e12 / alu_peak,
                "traffic": recorded_traffic(w.name, kernel_kind(w, launches)),
                "peak_source": "CUDA-core fp32 FMA, 148 SMs x 128 lanes x 2 flop x max SM "
                               "clock", "algorithmic_flops_per_launch": aflops,
                "kernel": "gdr_chunk_bwd"}
    else:
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak,
                "traffic": recorded_traffic(w.name, kernel_kind(w, launches)),
                "peak_source": peak_kind, "algorithmic_bytes_per_launch": abytes,
                "kernel": ("gdr_chunk_bwd (tensor cores, 3 launches)" if w.backward else
                           "gdr_chunk_fwd_prologue" if w.prologue else
                           "gdr_chunk_fwd_gla" if w.mixer == "gla" else
                           "gdr_dplr_fwd" if w.mixer == "dplr" else "gdr_chunk_fwd")
                if w.kind == "chunk" else "gdr_step"}
    return {"value": world * tokens_step * steps / (total_ms / 1e3), "ms_per_step": ms_step,
            "tflops": aflops * world * steps / (total_ms / 1e3) / 1e12,
            "roofline_time_ms": roof_ms, "roofline_fraction": roof_ms / ms_step,
            "roofline": roof, "tokens_step": tokens_step}


# The other workloads of the benchmark, timed in the same process after the
# headline one (one GPU): the long sequence (segment path), the per-channel
# gate, the decode step and the tiny fp32 forward.
EXTRA_WORKLOADS = ("gdn_b1_t65536_h16_d128", "kda_b8_t4096_h16_d128",
                   "decode_n256_h16_d128_x1024", "tiny_fp32")


def time_extra(name, args, rank, world, local_rank, dev):
    w = WORKLOADS[name]
    steps, warmup = max(5, min(args.steps, 20)), 3
    r = make_step(w, dev, rank, warmup + steps + 3)
    total_ms, per_launch, clk = time_device(r["step"], steps, warmup, dev, world, local_rank)
    f = roofline_fields(w, total_ms, per_launch, steps, world, clk, r["launches"])
    out = {"metric_value": f["value"], "unit": "tokens/s", "ms_per_step": f["ms_per_step"],
           "steps": steps, "warmup": warmup, "tflops": f["tflops"],
           "roofline_fraction": f["roofline_fraction"], "roofline": f["roofline"],
           "gpu_launches": steps * r["launches"], "clocks": clk,
           "config": {"B": w.B, "T": w.T if w.kind == "chunk" else 1, "H": w.H, "d_k": w.dk,
                      "d_v": w.dv, "gate": w.gate, "S0": w.with_S0, "S_T": w.want_S_T,
                      "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32"}}
    if w.kind == "step":
        out["config"]["note"] = ("one gdr_step over all 256 x 16 states per step; the state "
                                 "is updated in place (%d consecutive steps timed)" % steps)
    del r
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    r = make_step(w, dev, rank, args.warmup + args.steps + 3)
    step, host, d, o, S_T, S = r["step"], r["host"], r["d"], r["o"], r["S_T"], r["S"]
    launches_per_step = r["launches"]

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- device-timed region: inputs resident in HBM
    total_ms, per_launch_ms, clk = time_device(step, args.steps, args.warmup, dev, world,
                                               local_rank)

    # ---- end to end through the same API with host buffers (pinned)
    from gated_delta_rule_93_b200 import binding

    if w.kind == "step":
        # per step: that step's q, k, v, g, beta go host -> device, o comes back;
        # the state stays resident (it is the decoder's cache)
        pin = {k: host[k][0].pin_memory() for k in ("q", "k", "v", "g", "beta")}
        dev_in = {k: torch.empty_like(v, device=dev) for k, v in pin.items()}
    else:
        pin = {k: (v.pin_memory() if v is not None else None) for k, v in host.items()}
        dev_in = d
    # the step's results read back: o (and S_T), or every gradient
    results = r["results"]
    res_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in results]
    h2d = sum(v.numel() * v.element_size() for v in pin.values() if v is not None)
    d2h = sum(t.numel() * t.element_size() for t in res_h)

    def e2e_step():
        for kk, v in pin.items():
            if v is not None:
                dev_in[kk].copy_(v, non_blocking=True)
        if w.kind == "step":
            binding.step(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["g"], dev_in["beta"], S,
                         o=o)
        else:
            step()
        for hb, t in zip(res_h, results):
            hb.copy_(t, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)

    # ---- max over ranks
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device=dev)
    f = roofline_fields(w, total_ms, per_launch_ms, args.steps, world, clk, launches_per_step)

    # ---- the other workloads, each timed on its own after the headline one
    extras = {}
    if world == 1 and not args.no_extra and w.name == DEFAULT_WORKLOAD:
        del r, step, host, d, dev_in, pin, results, res_h
        torch.cuda.empty_cache()
        for name in EXTRA_WORKLOADS:
            extras[name] = time_extra(name, args, rank, world, local_rank, dev)

    if rank != 0:
        return None
    line = {
        "metric": METRIC,
        "value": f["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": f["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; q,k L2-normalised N(0,1), v N(0,1), "
                "beta=sigmoid(N(0,1)), log alpha=-0.1 softplus(N(0,1)))",
        "config": {"workload": w.name, "B": w.B, "T": w.T if w.kind == "chunk" else 1,
                   "H": w.H, "d_k": w.dk, "d_v": w.dv,
                   "chunk": w.C, "gate": w.gate, "S0": w.with_S0, "S_T": w.want_S_T,
                   "global_batch": w.B * world, "seq_len": w.T if w.kind == "chunk" else 1,
                   "parallelism": f"independent (b,h) shards x{world}",
                   "l2": "inputs exceed L2 (%.0f MB > 126 MB); no flush" %
                         (algorithmic_bytes(w) / 1e6)},
        "tflops": f["tflops"],
        "roofline_time_ms": f["roofline_time_ms"],
        "roofline_fraction": f["roofline_fraction"],
        "roofline": f["roofline"],
        "e2e": {"value": world * f["tokens_step"] * e2e_steps / (e2e_ms / 1e3),
                "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clk,
    }
    if extras:
        line["configs"] = extras
        line["gpu_launches_all"] = line["gpu_launches"] + sum(
            x["gpu_launches"] for x in extras.values())
    if rank == 0 and world == 1 and not args.no_cpu_baseline and w.kind == "chunk":
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return line


# ------------------------------------------------------------------ oracle arm
def _oracle_sample(w, inp, Tp):
    """The oracle's arguments for the first Tp tokens of every (b, h)."""
    from gated_delta_rule_93_b200.inputs import to_numpy_input

    sl = {k: (v[:, :Tp].contiguous() if (v is not None and k not in ("S0", "gate_scale"))
              else v) for k, v in inp.items()}
    S0 = None if sl["S0"] is None else sl["S0"].double().numpy()
    qkv = [to_numpy_input(sl["q"]), to_numpy_input(sl["k"]), to_numpy_input(sl["v"])]
    if w.prologue:
        return qkv + [sl["a"].numpy(), sl["b"].numpy(), sl["gate_scale"].numpy(), S0]
    if w.backward:
        return qkv + [sl["g"].numpy(), sl["beta"].numpy(), sl["dout"].double().numpy(), S0]
    if w.mixer == "dplr":
        return qkv + [to_numpy_input(sl["a"]), to_numpy_input(sl["b"]), sl["g"].numpy(), S0]
    return qkv + [sl["g"].numpy(), sl["beta"].numpy(), S0]


def _oracle_fwd(oracle, w, a, n):
    """The oracle's forward for the workload (arguments from _oracle_sample)."""
    if w.prologue:
        return oracle.gdr_fwd_prologue(*a, gate=w.gate, nthreads=n)
    if w.backward:
        return oracle.gdr_bwd(*a, gate=w.gate, nthreads=n)
    if w.mixer == "dplr":
        return oracle.dplr_fwd(*a, gate=w.gate, nthreads=n)
    if w.mixer == "gla":
        return oracle.gla_fwd(a[0], a[1], a[2], a[3], a[5], gate=w.gate, nthreads=n)
    return oracle.gdr_fwd(*a, gate=w.gate, nthreads=n)


def cpu_baseline(w, target_s=12.0):
    """Time the fp64 oracle, as it stands, on a bounded sample of the workload:
    all B*H heads over the first T' tokens, T' grown until a run takes a few
    seconds, then tokens/s = B*T'/elapsed."""
    import oracle
    from gated_delta_rule_93_b200.inputs import to_numpy_input

    oracle.build()
    inp = make_workload_inputs(w)
    n = min(oracle.default_threads(), w.B * w.H)
    # the oracle backward keeps every state of a head (2 x 128 KB per token at
    # d = 128, per thread): its sample stops at 512 tokens
    t_cap = min(w.T, 512) if w.backward else w.T
    Tp = 16
    while True:
        args = _oracle_sample(w, inp, Tp)
        t = time.perf_counter()
        _oracle_fwd(oracle, w, args, n)
        el = time.perf_counter() - t
        if el >= target_s / 4 or Tp >= t_cap:
            break
        Tp = min(t_cap, max(Tp * 2, int(Tp * (target_s / 3) / max(el, 1e-3))))
    return {"value": w.B * Tp / el, "unit": "tokens/s", "cores": n, "kind": "oracle",
            "sample": f"all {w.B}x{w.H} (b,h) pairs, first {Tp} of {w.T} tokens "
                      f"({el:.2f} s wall, fp64 C recurrence, {n} threads)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    import oracle
    from gated_delta_rule_93_b200.inputs import to_numpy_input

    oracle.build()
    inp = make_workload_inputs(w)
    n = min(oracle.default_threads(), w.B * w.H)
    # bounded per-step sample: first Tp tokens of every (b, h)
    Tp = max(1, min(w.T, args.ref_tokens))
    a = _oracle_sample(w, inp, Tp)
    for _ in range(args.warmup):
        _oracle_fwd(oracle, w, a, n)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_fwd(oracle, w, a, n)
    el = time.perf_counter() - t
    val = w.B * Tp * args.steps / el
    sample = (f"all {w.B}x{w.H} (b,h) pairs, first {Tp} of {w.T} tokens per step "
              f"(fp64 C recurrence, {n} threads)")
    return {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "d_k": w.dk,
                       "d_v": w.dv, "chunk": w.C, "gate": w.gate},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": n, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the chosen workload (not the other workloads after it)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-tokens", type=int, default=64)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
