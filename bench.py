"""Benchmark: causal linear attention prefill / decode on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one call of the hot path over one batch of the workload's synthetic input
(prefill: la_prefill over B x T tokens; decode: la_decode_step for N sequences).  The
default workload is the ungated elu+1 prefill (bf16, B=4, H=16, T=4096, d=128, chunk 64);
``--extras`` (default on at N=1) also measures the other three workloads and reports
them under "workloads".  Prints ONE JSON line on rank 0.

Under torchrun each rank runs its own copy of the workload on its own GPU (independent
sequences, no collective on the data path: weak scaling); the timed region is bracketed
by a barrier and a device synchronise, and the max over ranks is reported.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload
(the only other place this file runs the oracle is the cpu_baseline leg).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "gdn_bf16_b2h16t32768"
METRIC = "prefill tokens/s + % tensor roofline; decode tokens/s + HBM GB/s (1×B200)"
L2_FLUSH_BYTES = 256 << 20          # > 126 MB L2
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(dist, device):
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------------
# workload accounting (algorithmic work, not what a kernel happens to do)
# ----------------------------------------------------------------------------------

def io_bytes(dtype):
    return 2 if dtype == torch.bfloat16 else 4


def prefill_algorithmic(w: W.Workload, C=64):
    """Bytes that must cross HBM once and flops of the chunked form at chunk C = 64.

    bytes: q, k, v read + o written, gates/beta read (mode 3: d_k gates per token),
    final state (and z) written.
    flops per token-head: modes 0/1/4  2C d_k + 2C d_v + 4 d_k d_v;
                          modes 2/3    10 C d + 6 d^2 + C^2 / 3  (d = d_k = d_v; the per-channel
                          decays of mode 3 are exponentials inside the products, not counted)."""
    th = w.B * w.H * w.T
    e = io_bytes(w.dtype)
    b = th * e * (2 * w.dk + 2 * w.dv)
    if w.gate == "softplus":   # per-token gates ("retnet": one constant per head, no stream)
        b += th * 4 * (w.dk if w.mode == 3 else 1)
    if w.beta:
        b += th * 4
    b += w.B * w.H * (w.dv * w.dk * 4 + (w.dk * 4 if w.mode == 0 else 0))
    if w.mode in (2, 3):   # the delta rule (mode 4 is the scalar-gate recurrence)
        d = w.dk
        f = 10 * C * d + 6 * d * d + C * C / 3.0
    else:
        f = 2 * C * w.dk + 2 * C * w.dv + 4 * w.dk * w.dv
    return float(b), float(th * f)


def decode_algorithmic(w: W.Workload):
    """Per decode step: state read + write (fp32), q,k,v read, o written, a/beta read."""
    nh = w.B * w.H
    e = io_bytes(w.dtype)
    b = nh * (2 * w.dk * w.dv * 4 + e * (2 * w.dk + 2 * w.dv))
    if w.gate != "none":
        b += nh * 4 * (w.dk if w.mode == 3 else 1)
    if w.beta:
        b += nh * 4
    if w.mode == 0:
        b += nh * 2 * w.dk * 4
    f = nh * 8 * w.dk * w.dv
    return float(b), float(f)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def kernel_sources_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_attention_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def source_file_shas():
    """{file: sha} of every kernel source file (csrc/*.cu, *.cuh)."""
    csrc = os.path.join(ROOT, "gated_delta_rule_attention_b200", "csrc")
    out = {}
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, fn), "rb") as f:
                out[fn] = hashlib.sha256(f.read()).hexdigest()[:16]
    return out


def ncu_traffic(workload: str):
    """The committed ncu launch summary of `workload` (kernels in launch order, each with
    its DRAM bytes per launch and time share), or None when a source file it was taken on
    has changed since.  An entry lists the files its kernels were built from (their
    translation units, every header, the C ABI); an entry without its own list is checked
    against every file recorded for the whole summary."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        now = source_file_shas()
        entry = t["workloads"][workload]
        rec = entry.get("sources") or t.get("sources")
        if not rec or any(now.get(fn) != sha for fn, sha in rec.items()):
            return None
        return entry
    except Exception:
        return None


# ----------------------------------------------------------------------------------
# clocks during the timed region (NVML, the library nvidia-smi reads)
# ----------------------------------------------------------------------------------

class ClockSampler:
    BAD = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
           "hw_power_brake_slowdown": 0x80}
    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
             0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = device_index
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                idx = int(vis.split(",")[device_index])
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        reasons = [n for bit, n in self.NAMES.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------------------------
# one workload on one GPU
# ----------------------------------------------------------------------------------

class PrefillCase:
    def __init__(self, la, w: W.Workload, device, rank, workspace="auto"):
        self.la, self.w, self.device = la, w, device
        self.ws = workspace
        wr = W.variant(w, seed=w.seed + 1000 * rank)
        self.inp = W.prefill_inputs(wr, device=device)
        self.state = torch.empty(w.B, w.H, w.dv, w.dk, device=device)
        self.z = torch.empty(w.B, w.H, w.dk, device=device) if w.mode == 0 else None
        self.o = torch.empty(w.B, w.H, w.T, w.dv, device=device, dtype=w.dtype)
        self.tokens = w.B * w.T
        self.bytes, self.flops = prefill_algorithmic(w)
        self.kind = "prefill"

    def step(self):
        i = self.inp
        self.la.prefill(i["q"], i["k"], i["v"], mode=self.w.mode, gate=i["gate"], beta=i["beta"],
                        state=self.state, z=self.z, o=self.o, chunk=self.w.chunk,
                        init_state=False, workspace=self.ws)

    def e2e_setup(self):
        pin = lambda t: None if t is None else t.to("cpu").pin_memory()
        self.h_in = {k: pin(v) for k, v in self.inp.items() if k in ("q", "k", "v", "gate", "beta")}
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h_state = torch.empty(self.state.shape, dtype=torch.float32).pin_memory()
        self.h_z = None if self.z is None else torch.empty(self.z.shape).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values() if t is not None)
        self.d2h = self.h_o.numel() * self.h_o.element_size() + self.h_state.numel() * 4 + (
            0 if self.h_z is None else self.h_z.numel() * 4)

    def e2e_step(self):
        """Host buffers in, host buffers out: copies on the stream, then the ABI call."""
        h = self.h_in
        d = {k: (None if v is None else self.inp[k]) for k, v in h.items()}
        for k, v in h.items():
            if v is not None:
                d[k].copy_(v, non_blocking=True)
        self.la.prefill(d["q"], d["k"], d["v"], mode=self.w.mode, gate=d["gate"], beta=d["beta"],
                        state=self.state, z=self.z, o=self.o, chunk=self.w.chunk, init_state=False,
                        workspace=self.ws)
        self.h_o.copy_(self.o, non_blocking=True)
        self.h_state.copy_(self.state, non_blocking=True)
        if self.h_z is not None:
            self.h_z.copy_(self.z, non_blocking=True)


class DecodeCase:
    """One step = one la_decode_step over N sequences; the timed loop walks the
    pre-generated per-token inputs so that every step reads fresh q, k, v, a, beta."""

    def __init__(self, la, w: W.Workload, device, rank, steps_needed):
        self.la, self.w, self.device = la, w, device
        wr = W.variant(w, seed=w.seed + 1000 * rank)
        self.n_inputs = max(1, min(steps_needed, w.T))
        self.inp = W.decode_inputs(wr, steps=self.n_inputs, device=device)
        self.state = self.inp["state0"].clone()
        self.z = None if self.inp["z0"] is None else self.inp["z0"].clone()
        self.o = torch.empty(w.B, w.H, w.dv, device=device, dtype=w.dtype)
        self.t = 0
        self.tokens = w.B
        self.bytes, self.flops = decode_algorithmic(w)
        self.kind = "decode"

    def step(self):
        i, t = self.inp, self.t % self.n_inputs
        self.t += 1
        self.la.decode_step(i["q"][t], i["k"][t], i["v"][t], mode=self.w.mode, state=self.state,
                            gate=None if i["gate"] is None else i["gate"][t],
                            beta=None if i["beta"] is None else i["beta"][t], z=self.z, o=self.o)

    def e2e_setup(self):
        t0 = 0
        pin = lambda t: None if t is None else t[t0].to("cpu").pin_memory()
        self.h_in = {k: pin(self.inp[k]) for k in ("q", "k", "v", "gate", "beta")}
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values() if t is not None)
        self.d2h = self.h_o.numel() * self.h_o.element_size()
        self.d_in = {k: (None if v is None else torch.empty_like(v, device=self.device))
                     for k, v in self.h_in.items()}

    def e2e_step(self):
        """Per token: copy q, k, v, a, beta in from pinned host memory, step the resident
        state, copy o back (the state stays on the device, as in serving)."""
        for k, v in self.h_in.items():
            if v is not None:
                self.d_in[k].copy_(v, non_blocking=True)
        d = self.d_in
        self.la.decode_step(d["q"], d["k"], d["v"], mode=self.w.mode, state=self.state,
                            gate=d["gate"], beta=d["beta"], z=self.z, o=self.o)
        self.h_o.copy_(self.o, non_blocking=True)


class VarlenCase:
    """One step = one la_prefill_varlen call over a packed serving batch (sequences of
    mixed lengths, each with its own state)."""

    def __init__(self, la, vw: W.VarlenWorkload, device, rank):
        self.la, self.vw, self.device = la, vw, device
        w = W.variant(vw.base, seed=vw.base.seed + 1000 * rank)
        self.w = w
        self.L = vw.lengths()
        self.inp = W.varlen_inputs(w, self.L, device=device)
        N, T = len(self.L), sum(self.L)
        self.state = torch.empty(N, w.H, w.dv, w.dk, device=device)
        self.z = torch.empty(N, w.H, w.dk, device=device) if w.mode == 0 else None
        self.o = torch.empty(w.H, T, w.dv, device=device, dtype=w.dtype)
        self.tokens = T
        b_tok, f_tok = prefill_algorithmic(W.variant(w, B=1, T=T))
        # prefill_algorithmic counts one final state per (batch, head): add the other N-1
        self.bytes = b_tok + (N - 1) * w.H * (w.dv * w.dk * 4 + (w.dk * 4 if w.mode == 0 else 0))
        self.flops = f_tok
        self.kind = "prefill_varlen"

    def step(self):
        i = self.inp
        self.la.prefill_varlen(i["q"], i["k"], i["v"], i["cu"], mode=self.w.mode, gate=i["gate"],
                               beta=i["beta"], state=self.state, z=self.z, o=self.o,
                               init_state=False)

    def e2e_setup(self):
        pin = lambda t: None if t is None else t.to("cpu").pin_memory()
        self.h_in = {k: pin(self.inp[k]) for k in ("q", "k", "v", "gate", "beta", "cu")}
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h_state = torch.empty(self.state.shape, dtype=torch.float32).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values() if t is not None)
        self.d2h = self.h_o.numel() * self.h_o.element_size() + self.h_state.numel() * 4

    def e2e_step(self):
        for k, v in self.h_in.items():
            if v is not None:
                self.inp[k].copy_(v, non_blocking=True)
        self.step()
        self.h_o.copy_(self.o, non_blocking=True)
        self.h_state.copy_(self.state, non_blocking=True)


class BackwardCase:
    """One step = one backward call: la_prefill_backward (mode 1) or
    la_prefill_backward_delta (modes 2, 3): dq, dk, dv, the gate gradient (and the rate
    gradient of the delta rule) from output cotangents dO."""

    def __init__(self, la, w: W.Workload, device, rank):
        self.la, self.w, self.device = la, w, device
        wr = W.variant(w, seed=w.seed + 1000 * rank)
        self.inp = W.prefill_inputs(wr, device=device)
        g = torch.Generator(device=device).manual_seed(wr.seed + 1)
        self.dO = torch.randn(w.B, w.H, w.T, w.dv, generator=g, device=device).to(w.dtype)
        self.tokens = w.B * w.T
        th = w.B * w.H * w.T
        e = io_bytes(w.dtype)
        self.delta = w.mode in (2, 3)
        if not self.delta:
            # read q, k, v, dO and the gates; write dq, dk, dv and the gate gradient
            self.bytes = float(th * (e * (3 * w.dk + 4 * w.dv) + 8))
            # forward recompute of the states and four d_k x d_v products per token-head,
            # plus the chunk's score products (C = 32)
            self.flops = float(th * (10 * w.dk * w.dv + 8 * 32 * (w.dk + w.dv)))
        else:
            gw = 4 * (w.dk if w.mode == 3 else 1)
            # read q, k, v, dO, gates, b; write dq, dk, dv, the gate and rate gradients
            self.bytes = float(th * (e * (4 * w.dk + 3 * w.dv) + 2 * gw + 8))
            # per token-head: nine d_k x d_v products (forward states: E and the state update;
            # reverse: E, dE, dW, E H^T, the carried cotangent (2), dq) and the chunk's
            # C-wide products (C = 32: Gram, WY factors, dT, T^T dW, dq/dk score terms)
            self.flops = float(th * (2 * 9 * w.dk * w.dv + 2 * 32 * (12 * w.dk + 7 * w.dv)))
        self.kind = "backward"

    def _call(self):
        i = self.inp
        if self.delta:
            return self.la.prefill_backward_delta(i["q"], i["k"], i["v"], self.dO, mode=self.w.mode,
                                                  beta=i["beta"], gate=i["gate"])[:3]
        return self.la.prefill_backward(i["q"], i["k"], i["v"], self.dO, mode=self.w.mode,
                                        gate=i["gate"])[:3]

    def step(self):
        self._call()

    def e2e_setup(self):
        pin = lambda t: t.to("cpu").pin_memory()
        self.h_in = {k: pin(self.inp[k]) for k in ("q", "k", "v", "gate") + (("beta",) if self.delta else ())}
        self.h_do = pin(self.dO)
        self.h_out = [torch.empty(self.inp["q"].shape, dtype=self.w.dtype).pin_memory() for _ in range(3)]
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in.values()) + \
            self.h_do.numel() * self.h_do.element_size()
        self.d2h = sum(t.numel() * t.element_size() for t in self.h_out)

    def e2e_step(self):
        for k, v in self.h_in.items():
            self.inp[k].copy_(v, non_blocking=True)
        self.dO.copy_(self.h_do, non_blocking=True)
        dq, dk, dv = self._call()
        for h, d in zip(self.h_out, (dq, dk, dv)):
            h.copy_(d, non_blocking=True)


class ConvCase:
    """One step = the short convolution prologue of one prefill batch: three
    la_short_conv calls (q and k with SiLU and the L2 norm, v with SiLU), token-major
    projections in, head-major attention inputs out."""

    def __init__(self, la, cw: W.ConvWorkload, device, rank):
        self.la, self.w, self.device = la, cw, device
        self.dims = [cw.dk, cw.dk, cw.dv]
        self.x, self.wt, self.y, self.win = [], [], [], []
        for i, d in enumerate(self.dims):
            C = cw.H * d
            x, w, _ = W.conv_inputs(cw.B, cw.T, C, cw.width, cw.dtype,
                                    seed=cw.seed + 10 * i + 1000 * rank, device=device, window=False)
            self.x.append(x)
            self.wt.append(w)
            self.y.append(torch.empty(cw.B, cw.H, cw.T, d, device=device, dtype=cw.dtype))
            self.win.append(torch.empty(cw.B, cw.width - 1, C, device=device, dtype=cw.dtype))
        self.tokens = cw.B * cw.T
        e = io_bytes(cw.dtype)
        self.bytes = float(sum(2 * cw.B * cw.T * cw.H * d * e + cw.H * d * cw.width * 4
                               + cw.B * (cw.width - 1) * cw.H * d * e for d in self.dims))
        self.flops = float(sum(2 * cw.width * cw.B * cw.T * cw.H * d for d in self.dims))
        self.kind = "conv"

    def _calls(self, collect=None):
        for i in range(3):
            self.la.short_conv(self.x[i], self.wt[i], heads=self.w.H, window_out=self.win[i],
                               silu=self.w.silu, l2norm=self.w.l2norm_qk and i < 2, y=self.y[i])
            if collect is not None:
                collect.extend(self.la.launch_times())

    def step(self):
        self._calls()

    def step_collect(self):
        out = []
        self._calls(out)
        return out

    def e2e_setup(self):
        self.h_x = [x.to("cpu").pin_memory() for x in self.x]
        self.h_y = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in self.y]
        self.h2d = sum(x.numel() * x.element_size() for x in self.h_x)
        self.d2h = sum(y.numel() * y.element_size() for y in self.h_y)

    def e2e_step(self):
        for hx, x in zip(self.h_x, self.x):
            x.copy_(hx, non_blocking=True)
        self._calls()
        for hy, y in zip(self.h_y, self.y):
            hy.copy_(y, non_blocking=True)


def time_steps(case, steps, warmup, dist, device, flush, fn=None, sampler=None):
    """Device time of `steps` calls of fn (default case.step), each bracketed by CUDA events
    on the launching stream, with an L2 flush between steps (outside the events)."""
    fn = fn or case.step
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(device)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    n0 = case.la.kernel_launches()
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            fn()
            ends[i].record(stream)
        torch.cuda.synchronize(device)
    launches = case.la.kernel_launches() - n0
    barrier(dist, device)
    torch.cuda.synchronize(device)
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return ms, launches


def launch_profile(case, steps, flush):
    """Device duration (ms) of each launch of one call, averaged over `steps` further
    calls: the library records CUDA events around each of its launches on the launching
    stream (la_launch_timing).  L2 is flushed between calls as in the timed region."""
    la = case.la
    la.launch_timing(True)
    per = []
    try:
        for _ in range(steps):
            if flush is not None:
                flush.zero_()
            if hasattr(case, "step_collect"):
                per.append(case.step_collect())
            else:
                case.step()
                per.append(la.launch_times())
    finally:
        la.launch_timing(False)
    n = min(len(p) for p in per) if per else 0
    return [statistics.mean(p[i] for p in per) for i in range(n)]


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def roofline(case, kernel_ms, step_ms, peaks, peak_src, prof):
    """Roofline of the call's outputs pass (its last launch, the one that reads and writes
    every token of the call: algorithmic bytes = the whole call's), timed by CUDA events on
    the launching stream, next to the same figure for the whole call (all launches)."""
    hbm_bound = case.bytes / (peaks["hbm_gbs"] * 1e9) >= case.flops / (peaks["bf16_tflops"] * 1e12)
    n = len(kernel_ms)
    names = ([k["name"] for k in prof["kernels"]] if prof and len(prof["kernels"]) == n
             else [f"launch {i}" for i in range(n)])
    t_call = (sum(kernel_ms) if n else step_ms) * 1e-3
    # a backward call splits its work over sweeps that each do a share of it: the whole call
    t_k = t_call if case.kind == "backward" else (kernel_ms[-1] if n else step_ms) * 1e-3
    if hbm_bound:
        unit, peak, work, scale = "GB/s", peaks["hbm_gbs"], case.bytes, 1e9
    else:
        unit, peak, work, scale = "TFLOP/s", peaks["bf16_tflops"], case.flops, 1e12
    ach = work / t_k / scale
    ach_call = work / t_call / scale
    traffic = None
    if prof and len(prof["kernels"]) == n and n:
        traffic = float(prof["kernels"][-1]["dram_bytes_per_launch"])
    return {
        "bound": "hbm" if hbm_bound else "tensor",
        "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak, "traffic": traffic,
        "kernel": (names[-1] if n and case.kind != "backward" else "call"),
        "kernel_ms": t_k * 1e3,
        "kernel_share": (t_k / t_call) if n else 1.0,
        "algorithmic_bytes": case.bytes, "algorithmic_flops": case.flops,
        "tensor_frac": case.flops / t_k / 1e12 / peaks["bf16_tflops"],
        "call": {"launches": n, "kernels": names, "kernel_ms": kernel_ms,
                 "achieved": ach_call, "frac": ach_call / peak,
                 "traffic": float(prof["dram_bytes_per_call"]) if prof else None},
        "peak_source": (f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"),
    }


def _sig(x, n=3):
    """x rounded to n significant digits (JSON-compact)."""
    if x is None or not math.isfinite(x) or x == 0:
        return x
    return float(f"{x:.{n}g}")


def compact(res, roof, cpu):
    """One short entry per extra workload (the driver keeps the end of the line): ms per
    step, tokens/s, the step's roofline fraction (algorithmic bytes or flops over the device
    time of all its launches), its tensor fraction, DRAM traffic per step over the
    algorithmic bytes (ncu, null when stale), the oracle's tokens/s on the host cores and
    the end-to-end tokens/s through host buffers."""
    tr = roof["call"]["traffic"]
    t_call = sum(roof["call"]["kernel_ms"]) * 1e-3 if roof["call"]["kernel_ms"] else None
    tc = res["algorithmic_flops_per_step"] / t_call / 1e12 / load_peaks()[0]["bf16_tflops"] if t_call else None
    return {"ms": _sig(res["ms_per_step"]), "tok_s": _sig(res["tokens_per_s"]),
            "frac": _sig(roof["call"]["frac"]), "tc": _sig(tc),
            "tx": _sig(tr / roof["algorithmic_bytes"]) if tr else None,
            "cpu": _sig(cpu["value"]) if cpu and cpu.get("value") else None,
            "e2e": _sig(res["e2e"]["value"]) if res.get("e2e") else None}


class LayerCase:
    """One step = a Gated DeltaNet layer's attention path from its projections: the short
    convolution of q, k, v (SiLU, q/k L2 norm) and the gated-delta prefill, either fused
    (la_prefill_conv) or as three la_short_conv calls and la_prefill."""

    def __init__(self, la, lw: W.LayerWorkload, device, rank):
        self.la, self.lw, self.device = la, lw, device
        cw, pw = lw.conv, lw.prefill
        self.x, self.wt = [], []
        for i in range(3):
            x, w, _ = W.conv_inputs(cw.B, cw.T, cw.H * 128, cw.width, cw.dtype,
                                    seed=cw.seed + 10 * i + 1000 * rank, device=device, window=False)
            self.x.append(x)
            self.wt.append(w)
        inp = W.prefill_inputs(W.variant(pw, seed=pw.seed + 1000 * rank), device=device)
        self.gate, self.beta = inp["gate"], inp["beta"]
        del inp
        B, H, T = cw.B, cw.H, cw.T
        self.y = torch.empty(3, B, H, T, 128, device=device, dtype=cw.dtype)
        self.win = torch.empty(3, B, cw.width - 1, H * 128, device=device, dtype=cw.dtype)
        self.o = torch.empty(B, H, T, 128, device=device, dtype=cw.dtype)
        self.state = torch.empty(B, H, 128, 128, device=device)
        self.tokens = lw.tokens
        pb, pf = prefill_algorithmic(pw)
        e = io_bytes(cw.dtype)
        th = B * H * T * 128
        # projections in, convolved q, k, v out (the layer's backward takes them), then the
        # prefill's bytes without its q, k, v reads (they are the rows just written)
        self.bytes = float(3 * th * e + 3 * th * e + pb - 3 * th * e
                           + 3 * (H * 128 * cw.width * 4 + B * (cw.width - 1) * H * 128 * e))
        self.flops = float(3 * 2 * cw.width * th + pf)
        self.kind = "layer"

    def _call(self, x, collect=None):
        la, cw = self.la, self.lw.conv
        if self.lw.fused:
            la.prefill_conv(*x, *self.wt, heads=cw.H, gate=self.gate, beta=self.beta, window_out=self.win,
                            y=self.y, o=self.o, state=self.state, init_state=False)
            if collect is not None:
                collect.extend(la.launch_times())
            return
        for i in range(3):
            la.short_conv(x[i], self.wt[i], heads=cw.H, window_out=self.win[i], silu=cw.silu,
                          l2norm=cw.l2norm_qk and i < 2, y=self.y[i])
            if collect is not None:
                collect.extend(la.launch_times())
        la.prefill(self.y[0], self.y[1], self.y[2], mode=2, gate=self.gate, beta=self.beta,
                   state=self.state, o=self.o, init_state=False, workspace="auto")
        if collect is not None:
            collect.extend(la.launch_times())

    def step(self):
        self._call(self.x)

    def step_collect(self):
        out = []
        self._call(self.x, out)
        return out

    def e2e_setup(self):
        self.h_x = [x.to("cpu").pin_memory() for x in self.x]
        self.h_g = [t.to("cpu").pin_memory() for t in (self.gate, self.beta)]
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_x + self.h_g)
        self.d2h = self.h_o.numel() * self.h_o.element_size()

    def e2e_step(self):
        for hx, x in zip(self.h_x, self.x):
            x.copy_(hx, non_blocking=True)
        self.gate.copy_(self.h_g[0], non_blocking=True)
        self.beta.copy_(self.h_g[1], non_blocking=True)
        self._call(self.x)
        self.h_o.copy_(self.o, non_blocking=True)


def measure(la, name, args, dist, device, rank, world, flush, with_e2e, sampler=None):
    if name in W.LAYER_CONFIGS:
        case = LayerCase(la, W.LAYER_CONFIGS[name], device, rank)
    elif name in W.CONV_CONFIGS:
        case = ConvCase(la, W.CONV_CONFIGS[name], device, rank)
    elif name in W.VARLEN_CONFIGS:
        case = VarlenCase(la, W.VARLEN_CONFIGS[name], device, rank)
    elif name in W.BACKWARD_CONFIGS:
        case = BackwardCase(la, W.BACKWARD_CONFIGS[name], device, rank)
    else:
        w = W.CONFIGS[name]
        case = (DecodeCase(la, w, device, rank, args.warmup + args.steps) if w.decode
                else PrefillCase(la, w, device, rank, None if args.no_workspace else "auto"))
    ms, launches = time_steps(case, args.steps, args.warmup, dist, device, flush, sampler=sampler)
    la.check_status()
    kernel_ms = launch_profile(case, args.steps, flush)
    total_ms = max_over_ranks(dist, sum(ms), device)
    tokens_all = sum_over_ranks(dist, case.tokens * args.steps, device)
    per_launch_ms = statistics.mean(ms) / max(1, launches // max(1, args.steps))
    peaks, peak_src = load_peaks()
    achieved_gbs = case.bytes / (statistics.mean(ms) * 1e-3) / 1e9
    achieved_tflops = case.flops / (statistics.mean(ms) * 1e-3) / 1e12
    res = {
        "workload": name,
        "tokens_per_s": tokens_all / (total_ms * 1e-3),
        "ms_per_step": total_ms / args.steps,
        "ms_per_step_median": statistics.median(ms),
        "launches_per_step": launches / args.steps,
        "algorithmic_bytes_per_step": case.bytes,
        "algorithmic_flops_per_step": case.flops,
        "hbm_gbs": achieved_gbs,
        "hbm_frac": achieved_gbs / peaks["hbm_gbs"],
        "tensor_tflops": achieved_tflops,
        "tensor_frac": achieved_tflops / peaks["bf16_tflops"],
        "attainable_frac": max(case.bytes / (peaks["hbm_gbs"] * 1e9),
                               case.flops / (peaks["bf16_tflops"] * 1e12)) / (statistics.mean(ms) * 1e-3),
        "peak_source": peak_src,
        "kernel_ms": kernel_ms,
        "_case": case, "_ms": ms, "_launches": launches, "_per_launch_ms": per_launch_ms,
    }
    if with_e2e:
        case.e2e_setup()
        e_ms, _ = time_steps(case, max(3, args.steps // 2), 2, dist, device, None, fn=case.e2e_step)
        e_total = max_over_ranks(dist, sum(e_ms), device)
        e_tokens = sum_over_ranks(dist, case.tokens * len(e_ms), device)
        res["e2e"] = {"value": e_tokens / (e_total * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": int(case.h2d), "d2h_bytes_per_step": int(case.d2h)}
    return res


# ----------------------------------------------------------------------------------
# the oracle on host cores
# ----------------------------------------------------------------------------------

def _timed_growing(run, n0, n_max, budget_s):
    """Call run(n) for n = n0, 2 n0, ... until one call takes half the budget or n_max is
    reached; returns (n, seconds of the last call)."""
    n = min(n0, n_max)
    while True:
        t0 = time.perf_counter()
        run(n)
        el = time.perf_counter() - t0
        if el * 2 > budget_s or n >= n_max:
            return n, el
        n = min(n_max, n * 2)


def oracle_sample_other(name, budget_s):
    """The oracle timed on a bounded sample of a convolution, packed-sequence or backward
    workload (tokens/s in the workload's token unit)."""
    import oracle
    f = lambda t: None if t is None else t.to(torch.float64).numpy()
    if name in W.CONV_CONFIGS:
        from oracle import conv as oc
        cw = W.CONV_CONFIGS[name]
        x, wt, _ = W.conv_inputs(1, min(cw.T, 4096), cw.H * cw.dk, cw.width, cw.dtype, seed=cw.seed,
                                 window=False)
        xs, ws_ = f(x), f(wt)
        T, el = _timed_growing(lambda n: oc.short_conv(xs[:, :n], ws_, H=cw.H, silu=cw.silu,
                                                       l2norm=cw.l2norm_qk), 256, xs.shape[1], budget_s)
        # one token = the three projections q, k, v
        return {"value": T / el / 3, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": f"1 x {T} tokens of one {cw.H}x{cw.dk} projection (fp64 numpy), /3"}
    if name in W.LAYER_CONFIGS:
        from oracle import conv as oc
        lw = W.LAYER_CONFIGS[name]
        cw = lw.conv
        xs = [f(W.conv_inputs(1, 512, 128, cw.width, cw.dtype, seed=cw.seed + i, window=False)[0]) for i in range(3)]
        ws_ = [f(W.conv_inputs(1, 1, 128, cw.width, cw.dtype, seed=cw.seed + i, window=False)[1]) for i in range(3)]
        inp = W.prefill_inputs(W.variant(lw.prefill, B=1, H=1, T=512), device="cpu")

        def run(n):
            ys = [oc.short_conv(xs[i][:, :n], ws_[i], H=1, silu=cw.silu, l2norm=cw.l2norm_qk and i < 2)[0]
                  for i in range(3)]
            oracle.prefill(2, ys[0], ys[1], ys[2], f(inp["gate"])[:, :, :n], f(inp["beta"])[:, :, :n])
        T, el = _timed_growing(run, 64, 512, budget_s)
        return {"value": T / el / cw.H, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                "sample": f"1 head x {T} tokens: fp64 convolution (numpy) then the fp64 C recurrence, /{cw.H} heads"}
    if name in W.VARLEN_CONFIGS:
        vw = W.VARLEN_CONFIGS[name]
        L = sorted(vw.lengths())[: max(2, vw.N // 8)]
        inp = W.varlen_inputs(vw.base, L, device="cpu")
        a = {k: f(inp[k]) for k in ("q", "k", "v", "gate", "beta")}
        cu = inp["cu"].numpy()
        t0 = time.perf_counter()
        oracle.prefill_packed(vw.base.mode, a["q"], a["k"], a["v"], cu, a["gate"], a["beta"])
        el = time.perf_counter() - t0
        return {"value": sum(L) / el, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
                "sample": f"the {len(L)} shortest sequences ({sum(L)} tokens) x {vw.base.H} heads "
                          f"(fp64 C, OpenMP)"}
    if name in W.BACKWARD_CONFIGS:
        from oracle import backward as ob
        w = W.BACKWARD_CONFIGS[name]
        inp = W.prefill_inputs(W.variant(w, B=1, H=min(w.H, 4), T=256), device="cpu")
        a = {k: f(inp[k]) for k in ("q", "k", "v", "gate") + (("beta",) if w.mode in (2, 3) else ())}
        do = np.random.default_rng(0).standard_normal(a["v"].shape)
        if w.mode in (2, 3):
            run = lambda n: ob.delta_backward(w.mode, a["q"][:, :, :n], a["k"][:, :, :n], a["v"][:, :, :n],
                                              a["gate"][:, :, :n], a["beta"][:, :, :n], do[:, :, :n])
        else:
            run = lambda n: ob.prefill_backward(w.mode, a["q"][:, :, :n], a["k"][:, :, :n], a["v"][:, :, :n],
                                                a["gate"][:, :, :n], do[:, :, :n])
        T, el = _timed_growing(run, 32, 256, budget_s)
        hs = a["q"].shape[1]
        return {"value": hs * T / el / w.H, "unit": "tokens/s", "cores": torch.get_num_threads(),
                "kind": "oracle", "sample": f"{hs} heads x {T} tokens (fp64 PyTorch autograd on the CPU)"}
    return None


def oracle_sample(name, budget_s=10.0):
    """Time the fp64 oracle on a bounded sample of the workload.  Returns a dict with
    tokens/s (in the workload's token unit), the cores used and a description."""
    import numpy as np
    import oracle
    if name not in W.CONFIGS:
        return oracle_sample_other(name, budget_s)
    w = W.CONFIGS[name]
    threads = oracle.max_threads()
    gen_w = W.variant(w, B=1, H=min(w.H, max(1, threads)), T=min(w.T, 4096) if not w.decode else w.T)
    if w.decode:
        inp = W.decode_inputs(w, steps=1, device="cpu", n_seqs=max(1, threads // w.H + 1))
        f = lambda t: None if t is None else t.to(torch.float64).numpy()
        q, k, v = f(inp["q"][0]), f(inp["k"][0]), f(inp["v"][0])
        g, b = f(inp["gate"][0]) if inp["gate"] is not None else None, f(inp["beta"][0]) if inp["beta"] is not None else None
        S = f(inp["state0"])
        z = f(inp["z0"]) if inp["z0"] is not None else None
        n_seq = q.shape[0]
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle.decode_step(w.mode, q, k, v, g, b, S, z)
            reps += 1
            el = time.perf_counter() - t0
            if el >= budget_s or reps >= 10000:
                break
        return {"value": reps * n_seq / el, "unit": "tokens/s", "cores": min(threads, n_seq * w.H),
                "kind": "oracle",
                "sample": f"{reps} decode steps of {n_seq} sequences x {w.H} heads (fp64 C, OpenMP)"}
    inp = W.prefill_inputs(gen_w, device="cpu")
    f = lambda t: None if t is None else t.to(torch.float64).numpy()
    args = [f(inp[x]) for x in ("q", "k", "v", "gate", "beta")]
    # time growing prefixes until the budget is reached
    T = min(256, gen_w.T)
    el = 0.0
    while True:
        sl = [None if a is None else (a if a.ndim == 1 else a[:, :, :T]) for a in args]
        t0 = time.perf_counter()
        oracle.prefill(w.mode, *sl)
        el = time.perf_counter() - t0
        if el * 2 > budget_s or T >= gen_w.T:
            break
        T = min(gen_w.T, T * 2)
    heads = gen_w.H
    token_heads_per_s = heads * T / el
    return {"value": token_heads_per_s / w.H, "unit": "tokens/s", "cores": min(threads, heads),
            "kind": "oracle",
            "sample": f"{heads} heads x {T} tokens of the workload's recipe (fp64 recurrent C, "
                      f"OpenMP over heads); tokens/s counts all {w.H} heads of a token"}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    name = args.workload
    if name not in W.CONFIGS:
        print(json.dumps({"impl": "reference", "unavailable": f"no oracle sample for {name}"}))
        return 0
    per_step = []
    res = None
    for i in range(args.warmup + args.steps):
        res = oracle_sample(name, budget_s=max(0.5, min(5.0, 120.0 / (args.warmup + args.steps))))
        if i >= args.warmup:
            per_step.append(res["value"])
    value = statistics.mean(per_step)
    w = W.CONFIGS[name]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": (w.tokens / value) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": name, "mode": w.mode, "B": w.B, "H": w.H, "T": w.T, "d_k": w.dk,
                   "d_v": w.dv, "io_dtype": str(w.dtype).replace("torch.", ""),
                   "parallelism": "host cores (OpenMP over heads)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": res["cores"],
                         "kind": "oracle", "sample": res["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------------

def workload_config(name, world):
    """(I/O dtype, the JSON line's config) of a workload of any of the three kinds."""
    common = {"parallelism": f"dp{world} (independent sequences per GPU)",
              "l2": "flushed between timed steps (256 MiB write)"}
    if name in W.CONV_CONFIGS:
        cw = W.CONV_CONFIGS[name]
        return cw.dtype, {"workload": name, "kind": "short convolution of q, k, v", "B": cw.B,
                          "H": cw.H, "T": cw.T, "d_k": cw.dk, "d_v": cw.dv, "width": cw.width,
                          "silu": cw.silu, "l2norm_qk": cw.l2norm_qk, "global_batch": cw.B * world,
                          "seq_len": cw.T, **common}
    if name in W.LAYER_CONFIGS:
        lw = W.LAYER_CONFIGS[name]
        cw = lw.conv
        return cw.dtype, {"workload": name, "kind": "short convolution + gated-delta prefill ("
                          + ("fused" if lw.fused else "separate calls") + ")", "mode": 2, "B": cw.B,
                          "H": cw.H, "T": cw.T, "d_k": 128, "d_v": 128, "width": cw.width,
                          "global_batch": cw.B * world, "seq_len": cw.T, "state_dtype": "f32",
                          "accum": "f32", **common}
    if name in W.VARLEN_CONFIGS:
        vw = W.VARLEN_CONFIGS[name]
        L = vw.lengths()
        return vw.base.dtype, {"workload": name, "kind": "packed variable-length prefill",
                               "mode": vw.base.mode, "N": vw.N, "H": vw.base.H, "tokens": sum(L),
                               "min_len": min(L), "max_len": max(L), "d_k": vw.base.dk,
                               "d_v": vw.base.dv, "global_batch": vw.N * world,
                               "seq_len": max(L), "state_dtype": "f32", "accum": "f32", **common}
    w = W.CONFIGS[name] if name in W.CONFIGS else W.BACKWARD_CONFIGS[name]
    return w.dtype, {"workload": name, "mode": w.mode, "B": w.B, "H": w.H, "T": w.T,
                     "d_k": w.dk, "d_v": w.dv, "chunk": w.chunk or "default",
                     "global_batch": w.B * world, "seq_len": w.T, **common,
                     "state_dtype": "f32", "accum": "f32"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(list(W.CONFIGS) + list(W.CONV_CONFIGS) + list(W.VARLEN_CONFIGS) +
                                   list(W.BACKWARD_CONFIGS) + list(W.LAYER_CONFIGS)))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--extras", type=int, default=-1,
                    help="1: also measure the other workloads (default: on at N=1)")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-workspace", action="store_true",
                    help="prefill without the segment workspace (one kernel per call)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    world, rank, local = dist_env()
    if world > 1 and args.gpus != world:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    dist = init_dist(world, local)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    import gated_delta_rule_attention_b200 as la
    la.library()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    sampler = ClockSampler(local)
    main_res = measure(la, args.workload, args, dist, device, rank, world, flush, True,
                       sampler=sampler)
    extras = {}
    do_extras = (world == 1) if args.extras < 0 else bool(args.extras)
    if do_extras:
        peaks_x, src_x = load_peaks()
        for name in ("elu1_f32_small", "elu1_bf16_b4h16t4096", "gated_bf16_b8h16t8192",
                     "gdn_bf16_b2h16t32768", "gdn_decode_n256h32", "kda_bf16_b2h16t32768",
                     "kda_decode_n256h32", "conv_bf16_b2h16t32768", "gdn_varlen_bf16_n64h16",
                     "retnet_bf16_b8h16t8192", "gated_bwd_bf16_b4h16t4096", "gdn_bwd_bf16_b2h16t32768",
                     "gdn_layer_fused_bf16_b2h16t32768", "gdn_layer_split_bf16_b2h16t32768"):
            if name == args.workload:
                continue
            r = measure(la, name, args, dist, device, rank, world, flush, True)
            rf = roofline(r["_case"], r["kernel_ms"], statistics.mean(r["_ms"]), peaks_x, src_x,
                          ncu_traffic(name))
            cpu_x = None
            if rank == 0 and world == 1:
                try:
                    cpu_x = oracle_sample(name, budget_s=1.5)
                except Exception:
                    cpu_x = None
            extras[name] = compact(r, rf, cpu_x)
            del r
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1:
        try:
            cpu = oracle_sample(args.workload, budget_s=args.cpu_budget)
        except Exception as e:  # the oracle is optional context, never the measurement
            cpu = {"value": None, "error": str(e)[:200], "kind": "oracle"}

    peaks, peak_src = load_peaks()
    dtype, wconfig = workload_config(args.workload, world)
    case = main_res["_case"]
    mean_ms = statistics.mean(main_res["_ms"])
    roof = roofline(case, main_res["kernel_ms"], mean_ms, peaks, peak_src, ncu_traffic(args.workload))

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": main_res["tokens_per_s"],
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": main_res["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if dtype == torch.bfloat16 else "f32",
            "data": "synthetic",
            "config": wconfig,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": main_res.get("e2e"),
            "gpu_launches": int(main_res["_launches"]),
            "clocks": sampler.summary(),
            "workloads": extras,
        }
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
