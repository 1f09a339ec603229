#!/usr/bin/env python
"""Throughput of the micro-block FP4 quantizer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--units U]

The default workload is the largest one: the dual-scale round trip on a bf16
32768 x 4096 tensor (N(0,1) x LogNormal(0,1) per-token gain): block-Hadamard
rotation of size 512, per-128 FP32 group scale + per-16 E4M3 micro-scale,
E2M1 codes packed, then dequantize + inverse FWHT-512 back to bf16.  Other
workloads (``--workload``) time the remaining paths at their full sizes.

One step = U batches of the workload, each a full-size tensor, in phases: the
first kernel of the path over all U batches back to back, then the next kernel
over all U batches.  CUDA events at the phase boundaries give each kernel's
duration as a back-to-back loop of that kernel alone, inside the timed region;
U is sized so that one step is a few milliseconds.  The batches rotate over R
resident buffer sets whose total exceeds 4x the L2 cache, so no launch reads
data an earlier launch left in L2.

Metric: input GB/s = bf16 input bytes x U x steps / device time of the K timed
steps (CUDA events, max over ranks), inputs resident in HBM.  Each phase's U
calls are captured once into a CUDA graph (after a first round of direct calls)
and replayed every step, so that no per-call host work gaps the launches
(--no-graph: one C ABI call per launch).  Under torchrun
every rank quantizes its own batches (weak scaling; the path has no exchange
step).

The JSON line adds: the roofline of the dominant kernel (algorithmic bytes per
launch / its mean back-to-back duration in the timed steps, against the
measured HBM copy bandwidth), every kernel's mean duration, an end-to-end
figure through the public API with host buffers (per step: pinned host ->
device copy of one batch, the path, device -> host copy of its outputs, all
inside the timed region; consecutive batches overlap on three streams), the SM
clocks sampled during the timed region, and the CPU oracle timed on the host
as a baseline (rank 0, N = 1).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

MIB = 1 << 20
L2_BYTES = 126 * 10**6
METRIC = "input GB/s quantized to NVFP4/MXFP4 on 1 B200; % of HBM roofline"
STEP_BYTES = 24e9  # algorithmic bytes per step (about 4 ms at the HBM roofline)
WARM_S = 0.3  # minimum warm-up time (s)


# ----------------------------------------------------------------------------- workloads

def make_workload(name: str, rows: int = 0):
    """The workload `name` (at its full size, or with `rows` rows when given)."""
    wl = _make_workload(name)
    if rows and rows != wl["M"]:
        wl = _make_workload(name, rows)
        wl["desc"] += f" [{rows} rows]"
    return wl


def _make_workload(name: str, rows: int = 0):
    """Returns dict(desc, M, K, inputs(np), bytes_in, kernels=[(label, alg_bytes)], ...)."""
    if name == "mxfp4":
        M, K = rows or 4096, 4096
        return dict(name=name, M=M, K=K, fmt="MXFP4", had=0,
                    desc="mxfp4_4096x4096 quantize + dequantize round trip "
                         "(bf16 0.5*Student-t(3), block 32, E8M0)",
                    x=lambda: workloads.mxfp4_student_t(M, K, seed=2),
                    kernels=[("quantize", M * K * 2 + M * K // 2 + M * K // 32),
                             ("dequantize", M * K // 2 + M * K // 32 + M * K * 2)])
    if name == "nvfp4":
        M, K = rows or 256, 1024
        return dict(name=name, M=M, K=K, fmt="NVFP4", had=0,
                    desc="nvfp4_256x1024 quantize, dynamic tensor scale (N(0,1), 1% x20)",
                    x=lambda: workloads.nvfp4_outliers(M, K, seed=1),
                    kernels=[("amax+quantize", 2 * M * K * 2 + M * K // 2 + M * K // 16)],
                    launches=2)
    if name.startswith("hadamard"):
        n = int(name[len("hadamard"):] or 128)
        M, K = rows or 8192, 4096
        return dict(name=name, M=M, K=K, fmt="NVFP4", had=n,
                    desc=f"hadamard{n}+nvfp4_8192x4096 quantize, static tensor scale "
                         "(N(0,1), 64 channels x50)",
                    x=lambda: workloads.hadamard_channels(M, K, seed=3),
                    kernels=[("quantize", M * K * 2 + M * K // 2 + M * K // 16)])
    if name == "arc":
        M, K, S = rows or 8192, 4096, 256
        return dict(name=name, M=M, K=K, S=S, fmt="NVFP4", had=0,
                    desc="arc_8192x4096 reorder+RMSNorm+NVFP4+residual(S=256), static tensor scale",
                    x=lambda: workloads.arc_activations(M, K, seed=4, S=S),
                    kernels=[("arc", M * K * 2 + M * (K + S) // 2 + M * (K + S) // 16)])
    if name == "arc_mxfp4":
        M, K, S = rows or 8192, 4096, 256
        return dict(name=name, M=M, K=K, S=S, fmt="MXFP4", had=0,
                    desc="arc_mxfp4_8192x4096 reorder+RMSNorm+MXFP4+residual(S=256)",
                    x=lambda: workloads.arc_activations(M, K, seed=4, S=S),
                    kernels=[("arc", M * K * 2 + M * (K + S) // 2 + M * (K + S) // 32)])
    if name == "arc_int4":
        M, K, S = rows or 8192, 4096, 256
        return dict(name=name, M=M, K=K, S=S, fmt="INT4", had=0,
                    desc="arc_int4_8192x4096 reorder+RMSNorm+INT4+residual(S=256), static tensor scale",
                    x=lambda: workloads.arc_activations(M, K, seed=4, S=S),
                    kernels=[("arc", M * K * 2 + M * (K + S) // 2 + M * (K + S) // 16)])
    if name == "dual":
        M, K = rows or 32768, 4096
        return dict(name=name, M=M, K=K, fmt="DUAL", had=512,
                    desc="dual_fwht512_32768x4096 quantize + dequantize/inverse-FWHT round trip "
                         "(N(0,1) x LogNormal(0,1) per-token gain)",
                    x=lambda: workloads.dual_gain(M, K, seed=5),
                    kernels=[("quantize", M * K * 2 + M * K // 2 + M * K // 16 + M * K // 128 * 4),
                             ("dequantize", M * K // 2 + M * K // 16 + M * K // 128 * 4 + M * K * 2)])
    raise SystemExit(f"unknown workload {name}")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark(self):
        return time.time()

    def stop(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sel = [ln for (t, ln) in self.lines if t0 - 0.05 <= t <= t1 + 0.05] or [ln for _, ln in self.lines]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in sel:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def peaks_tensor():
    """Dense bf16 tensor TFLOP/s (burst figure) from MEASURED_PEAKS.json, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]) * 1e12, "measured"
    except (OSError, KeyError, ValueError):
        return 1590e12, "fallback"


# Source files each timed kernel is compiled from (the entry points' host code
# in fp4q.cu excluded): a committed ncu figure is used only while they are unchanged.
_COMMON = ["fp4q_device.cuh", "fp4q_unit.cuh", "fp4q_quant.cuh"]
KERNEL_SOURCES = {
    ("dual", "quantize"): _COMMON + ["fp4q_mma.cuh", "fp4q_mma_wide.cuh"],
    ("dual", "dequantize"): _COMMON + ["fp4q_mma.cuh", "fp4q_gemm.cuh", "fp4q_dqmma.cuh"],
    ("mxfp4", "quantize"): _COMMON,
    ("mxfp4", "dequantize"): _COMMON + ["fp4q_dequant.cuh"],
    ("hadamard128", "quantize"): _COMMON + ["fp4q_mma.cuh"],
    ("arc", "arc"): _COMMON + ["fp4q_arc.cuh"],
    ("arc_mxfp4", "arc"): _COMMON + ["fp4q_arc.cuh"],
    ("arc_int4", "arc"): _COMMON + ["fp4q_arc.cuh"],
}


def kernel_source_sha(files=None) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp4_micro_block_b200", "csrc")
    names = sorted(files) if files else sorted(fn for fn in os.listdir(csrc) if fn.endswith((".cu", ".cuh")))
    for fn in names:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel_label: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current sources of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}_{kernel_label}.txt")
    try:
        txt = open(path).read()
    except OSError:
        return None
    sha = re.search(r"source_sha:\s*(\w+)", txt)
    val = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not sha or not val or sha.group(1) != kernel_source_sha(KERNEL_SOURCES.get((workload, kernel_label))):
        return None
    return float(val.group(1))


# ----------------------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import torch
    import fp4_micro_block_b200 as fq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = make_workload(args.workload, args.rows)
    M, K = wl["M"], wl["K"]
    raw = wl["x"]()
    gamma_t = perm_t = outl_t = None
    if wl["name"].startswith("arc"):
        x_np, gamma, perm, outl = raw
        gamma_t = torch.from_numpy(gamma.view(np.int16)).view(torch.bfloat16).to(dev)
        perm_t = torch.from_numpy(perm).to(dev)
        outl_t = torch.from_numpy(outl).to(dev)
    else:
        x_np = raw
    x_host = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16)
    in_bytes = M * K * 2

    S = wl.get("S", 0)
    KS = K + S
    fmt = {"MXFP4": fq.FP4Q_MXFP4, "NVFP4": fq.FP4Q_NVFP4, "DUAL": fq.FP4Q_NVFP4_DUAL,
           "INT4": fq.FP4Q_INT4}[wl["fmt"]]
    B = 32 if fmt == fq.FP4Q_MXFP4 else 16
    labels = [k for k, _ in wl["kernels"]]
    alg = dict(wl["kernels"])
    has_dq = labels[-1] == "dequantize"
    set_bytes = in_bytes + M * KS // 2 + M * KS // B + (M * K * 2 if has_dq else 0)
    R = min(64, max(2, int(np.ceil(4 * L2_BYTES / set_bytes))))
    # batches per step: about STEP_BYTES of algorithmic traffic, so that a step
    # lasts a few milliseconds whatever the workload
    U = args.units or min(2048, max(R, int(np.ceil(STEP_BYTES / sum(alg.values())))))
    xs, outs = [], []
    for i in range(R):
        xi = x_host.to(dev)
        codes = torch.empty((M, KS // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty((M, KS // B), dtype=torch.uint8, device=dev)
        if fmt in (fq.FP4Q_NVFP4, fq.FP4Q_INT4):
            sf = torch.zeros(1, dtype=torch.float32, device=dev)
        elif fmt == fq.FP4Q_NVFP4_DUAL:
            sf = torch.empty((M, K // 128), dtype=torch.float32, device=dev)
        else:
            sf = None
        y = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if has_dq else None
        xs.append(xi)
        outs.append((codes, scales, sf, y))
    ws = fq.workspace(dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    L = fq.lib()

    # static tensor scale for the Hadamard / ARC workloads: the dynamic value of a first call
    if wl["name"].startswith("hadamard") or wl["name"] in ("arc", "arc_int4"):  # tensor scale
        for i in range(R):
            codes, scales, sf, _ = outs[i]
            if wl["name"].startswith("arc"):
                fq.fp4q_arc_quantize(xs[i], gamma_t, 1e-6, perm_t, outl_t, fmt, codes, scales, sf,
                                     fq.FP4Q_TSCALE_DYNAMIC, 0, ws)
            else:
                fq.fp4q_hadamard_quantize(xs[i], wl["had"], fmt, codes, scales, sf,
                                          fq.FP4Q_TSCALE_DYNAMIC, 0, ws)
        torch.cuda.synchronize()

    p = lambda t: None if t is None else t.data_ptr()

    def make_calls(i, sh):
        """One zero-arg callable per kernel label on buffer set i, enqueued on the
        stream whose handle is sh."""
        codes, scales, sf, y = outs[i]
        xp, cp, sp, fp, yp = p(xs[i]), p(codes), p(scales), p(sf), p(y)
        if wl["name"] == "mxfp4":
            return [lambda: L.fp4q_quantize_mxfp4(xp, M, K, K, cp, sp, 0, sh),
                    lambda: L.fp4q_dequantize(fq.FP4Q_MXFP4, cp, sp, None, M, K, 0, 0, yp, sh)]
        if wl["name"] == "nvfp4":
            return [lambda: L.fp4q_quantize_nvfp4(xp, M, K, K, cp, sp, fp, fq.FP4Q_TSCALE_DYNAMIC, 0,
                                                  ws.data_ptr(), fq.FP4Q_WORKSPACE_BYTES, sh)]
        if wl["name"].startswith("hadamard"):
            return [lambda: L.fp4q_hadamard_quantize(xp, M, K, K, wl["had"], fmt, cp, sp, fp,
                                                     fq.FP4Q_TSCALE_STATIC, 0, None, 0, sh)]
        if wl["name"].startswith("arc"):
            return [lambda: L.fp4q_arc_quantize(xp, M, K, K, gamma_t.data_ptr(), 1e-6, perm_t.data_ptr(),
                                                outl_t.data_ptr(), S, fmt, cp, sp, fp, fq.FP4Q_TSCALE_STATIC, 0,
                                                None, 0, sh)]
        return [lambda: L.fp4q_hadamard_quantize(xp, M, K, K, 512, fmt, cp, sp, fp, 0, 0, None, 0, sh),
                lambda: L.fp4q_dequantize(fmt, cp, sp, fp, M, K, 0, 512, yp, sh)]  # dual

    calls = [make_calls(i, sh) for i in range(R)]  # per buffer set
    # launches of our kernels per batch (the NVFP4 dynamic mode runs an amax
    # pre-pass and the quantizer inside one entry point)
    launches_per_batch = wl.get("launches", len(wl["kernels"]))
    n_lab = len(labels)

    graphs = None

    def step(evs=None):
        """U batches, one phase per kernel label; evs[j] is recorded before phase j."""
        for j in range(n_lab):
            if evs is not None:
                evs[j].record(stream)
            if graphs is not None:
                graphs[j].replay()
                continue
            for u in range(U):
                st = calls[u % R][j]()
                if st != 0:
                    raise RuntimeError(f"{labels[j]}: {fq.status_string(st)}")
        if evs is not None:
            evs[n_lab].record(stream)

    if args.graph:
        # Each phase's U calls captured once into a CUDA graph and replayed in
        # every step: the launches carry no per-call host work (argument checks,
        # tensor-map encoding, the ctypes call), as a serving loop would run them.
        step()  # first calls outside capture (per-device attributes, cached addresses)
        torch.cuda.synchronize()
        gs = torch.cuda.Stream(dev)
        gcalls = [make_calls(i, gs.cuda_stream) for i in range(R)]
        graphs_ = []
        for j in range(n_lab):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=gs, capture_error_mode="relaxed"):
                for u in range(U):
                    st = gcalls[u % R][j]()
                    if st != 0:
                        raise RuntimeError(f"{labels[j]} (capture): {fq.status_string(st)}")
            graphs_.append(g)
        graphs = graphs_
        torch.cuda.synchronize()

    dist = world > 1
    if dist:
        import torch.distributed as tdist

    # warm-up: W steps, continued until WARM_S seconds have passed (clocks and
    # caches settled); the same count on every rank
    t0 = time.perf_counter()
    n_warm = 0
    while n_warm < args.warmup or time.perf_counter() - t0 < WARM_S:
        step()
        torch.cuda.synchronize()
        n_warm += 1
    if dist:
        t = torch.tensor([n_warm], device=dev, dtype=torch.int64)
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        for _ in range(int(t.item()) - n_warm):
            step()
        n_warm = int(t.item())
    torch.cuda.synchronize()
    assert fq.fp4q_device_error() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_lab + 1)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    phys = int(vis[local_rank]) if len(vis) > local_rank and vis[local_rank].strip().isdigit() else local_rank
    sampler = ClockSampler(phys)
    sampler.start()
    if dist:
        tdist.barrier()
    torch.cuda.synchronize()
    w0 = sampler.mark()
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    w1 = sampler.mark()
    if dist:
        tdist.barrier()
    clocks = sampler.stop(w0, w1)
    assert fq.fp4q_device_error() == 0

    total_ms = t_start.elapsed_time(t_end)
    phase_ms = np.array([[evs[k][j].elapsed_time(evs[k][j + 1]) for j in range(n_lab)]
                         for k in range(args.steps)])
    if dist:
        t = torch.tensor([total_ms] + phase_ms.sum(axis=0).tolist(), device=dev, dtype=torch.float64)
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        total_ms = float(t[0].item())
        phase_tot = t[1:].cpu().numpy()
    else:
        phase_tot = phase_ms.sum(axis=0)
    # mean duration of one launch of each kernel in its back-to-back phase
    launch_us = {lab: float(phase_tot[j] / (args.steps * U) * 1e3) for j, lab in enumerate(labels)}
    dom = max(labels, key=lambda l: launch_us[l])
    achieved = alg[dom] / (launch_us[dom] * 1e-6) / 1e9
    peak, peak_src = peaks()
    value = in_bytes * U * args.steps * world / (total_ms * 1e-3) / 1e9

    # ---------------------------------------------------------------- end to end
    # Every step takes one batch through the public C ABI: the host -> device copy
    # of its input from pinned memory, the path, and the device -> host copy of
    # its outputs.  Consecutive batches overlap on three streams (inputs, path,
    # outputs) over two buffer sets, the way a caller streaming batches runs
    # them: PCIe moves one batch's outputs while it moves the next one's input.
    n_e2e = max(3, min(args.steps, 20))
    NB = min(2, R)
    x_pin = x_host.pin_memory()
    h_outs = [tuple(None if t is None else torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs[b])
              for b in range(NB)]
    d2h = sum(t.numel() * t.element_size() for t in outs[0] if t is not None)
    s_in, s_run, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    e2e_calls = [make_calls(b, s_run.cuda_stream) for b in range(NB)]
    ev_in, ev_run, ev_out = ([torch.cuda.Event() for _ in range(NB)] for _ in range(3))
    used = [False] * NB

    def e2e_step(k):
        b = k % NB
        if used[b]:
            s_in.wait_event(ev_run[b])  # the path of batch k - NB has read xs[b]
        with torch.cuda.stream(s_in):
            xs[b].copy_(x_pin, non_blocking=True)
        ev_in[b].record(s_in)
        s_run.wait_event(ev_in[b])
        if used[b]:
            s_run.wait_event(ev_out[b])  # the outputs of batch k - NB are on the host
        for j in range(n_lab):
            st = e2e_calls[b][j]()
            if st != 0:
                raise RuntimeError(f"{labels[j]}: {fq.status_string(st)}")
        ev_run[b].record(s_run)
        s_out.wait_event(ev_run[b])
        with torch.cuda.stream(s_out):
            for hd, dv in zip(h_outs[b], outs[b]):
                if hd is not None:
                    hd.copy_(dv, non_blocking=True)
        ev_out[b].record(s_out)
        used[b] = True

    for k in range(NB):
        e2e_step(k)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)  # every timed copy and launch follows it through the event chain
    for k in range(n_e2e):
        e2e_step(k)
    b.record(s_out)  # after the last batch's outputs
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b)
    if dist:
        t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e = {"value": round(in_bytes * n_e2e * world / (e2e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
           "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": int(d2h), "steps": n_e2e,
           "step": "one batch: host->device copy, the path through the C ABI, device->host copy; "
                   "consecutive batches overlap on three streams over two buffer sets"}
    assert fq.fp4q_device_error() == 0

    # ---------------------------------------------------------------- CPU oracle baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, x_np, raw, budget_s=args.cpu_budget)

    traffic = ncu_traffic(wl["name"], dom)
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl["desc"], "M": M, "K": K, "format": wl["fmt"],
                   "hadamard": wl["had"], "batches_per_step": U,
                   "per_rank_batch": f"{U}x{M}x{K} bf16 per step",
                   "global_batch": f"{world}x{U}x{M}x{K}",
                   "l2": f"inputs larger than L2; batches rotate over {R} buffer sets "
                         f"({R * set_bytes / MIB:.0f} MiB > 4x126 MB L2)",
                   "launch": "CUDA graph of each phase's calls" if graphs is not None
                             else "one C ABI call per launch",
                   "parallelism": f"dp{world}"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "peak_source": peak_src,
                     "alg_bytes_per_launch": alg[dom], "mean_launch_us": round(launch_us[dom], 3),
                     "timing": f"CUDA events around the {U} back-to-back launches of each phase, "
                               f"every timed step",
                     "frac_of_nominal_8000": round(achieved / 8000.0, 4)},
        "kernels_us": {lab: round(launch_us[lab], 3) for lab in labels},
        "kernels_frac": {lab: round(alg[lab] / (launch_us[lab] * 1e-6) / 1e9 / peak, 4) for lab in labels},
        "e2e": e2e,
        "gpu_launches": launches_per_batch * U * args.steps,
        "warmup_steps_run": n_warm,
        "clocks": clocks,
        "cpu_baseline": cpu,
        "impl": "ours",
    }
    return line


def run_arc_gemm(args, local_rank):
    """ARCQuant's cost on the consumer side: the fused ARC quantizer plus the
    block-scaled NVFP4 GEMM over K + S, against the same fused kernel without
    residual channels (S = 0) plus the GEMM over K.  Activations: the ARC
    workload (bf16 8192 x 4096, 256 outlier channels); weights: bf16
    N(0,1) 4096 x 4096 in the activations' channel order, quantized NVFP4 once
    outside the timed region ([W | W_S] for K + S).  Each kernel is timed as a
    back-to-back phase of U launches inside every step (CUDA events)."""
    import torch
    import fp4_micro_block_b200 as fq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, K, S, N = 8192, 4096, 256, 4096
    x_np, gamma, perm, outl = workloads.arc_activations(M, K, seed=4, S=S)
    rng = np.random.default_rng(7)
    w = workloads.to_bf16_bits(rng.standard_normal((N, K)))[:, perm]
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    g_t, p_t, o_t = bf(gamma), torch.from_numpy(perm).to(dev), torch.from_numpy(outl).to(dev)
    SW = fq.FP4Q_SCALES_SWIZZLED
    wb_aug = fq.quantize_nvfp4(bf(np.concatenate([w, w[:, outl]], axis=1)), None, SW)
    wb_k = fq.quantize_nvfp4(bf(w), None, SW)
    R = 4  # input sets: 4 x 64 MiB of activations > 2 x L2
    xs = [bf(x_np) for _ in range(R)]
    st = fq.arc_quantize(xs[0], g_t, p_t, o_t, 1e-6, None, SW)[2]  # calibrated s_t stand-in
    outs_aug = [fq.alloc_outputs(M, K + S, fq.FP4Q_NVFP4, SW, dev) for _ in range(R)]
    outs_k = [fq.alloc_outputs(M, K, fq.FP4Q_NVFP4, SW, dev) for _ in range(R)]
    for o in outs_aug + outs_k:
        o[2].copy_(st)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    L, sh = fq.lib(), torch.cuda.current_stream(dev).cuda_stream
    pp = lambda t: t.data_ptr()

    def arc(i, with_res):
        c, s_, sf = (outs_aug if with_res else outs_k)[i]
        return L.fp4q_arc_quantize(pp(xs[i]), M, K, K, pp(g_t), 1e-6, pp(p_t), pp(o_t) if with_res else None,
                                   S if with_res else 0, fq.FP4Q_NVFP4, pp(c), pp(s_), pp(sf),
                                   fq.FP4Q_TSCALE_STATIC, SW, None, 0, sh)

    def gemm(i, with_res):
        c, s_, sf = (outs_aug if with_res else outs_k)[i]
        wc, ws, wt = wb_aug if with_res else wb_k
        return L.fp4q_gemm_nvfp4(pp(c), pp(s_), pp(sf), pp(wc), pp(ws), pp(wt), M, N, K + S if with_res else K,
                                 pp(d), 1, sh)

    labels = ["arc_S256", "gemm_K4352", "arc_S0", "gemm_K4096"]
    fns = [lambda i: arc(i, True), lambda i: gemm(i, True), lambda i: arc(i, False), lambda i: gemm(i, False)]
    U = args.units or 16
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        for j, f in enumerate(fns):
            if evs is not None:
                evs[j].record(stream)
            for u in range(U):
                st_ = f(u % R)
                if st_ != 0:
                    raise RuntimeError(f"{labels[j]}: {fq.status_string(st_)}")
        if evs is not None:
            evs[len(fns)].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert fq.fp4q_device_error() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    sampler.start()
    torch.cuda.synchronize()
    w0 = sampler.mark()
    for k in range(args.steps):
        step(evs[k])
    torch.cuda.synchronize()
    clocks = sampler.stop(w0, sampler.mark())
    assert fq.fp4q_device_error() == 0
    us = {lab: float(np.sum([evs[k][j].elapsed_time(evs[k][j + 1]) for k in range(args.steps)])
                     / (args.steps * U) * 1e3) for j, lab in enumerate(labels)}
    flops = {"gemm_K4352": 2.0 * M * N * (K + S), "gemm_K4096": 2.0 * M * N * K}
    bf16_peak, src = peaks_tensor()
    fp4_peak = 4.0 * bf16_peak  # dense FP4 : bf16 tensor rate, 9 : 2.25 PFLOP/s nominal
    tf = {k: flops[k] / (us[k] * 1e-6) / 1e12 for k in flops}
    overhead = (us["arc_S256"] + us["gemm_K4352"]) / (us["arc_S0"] + us["gemm_K4096"]) - 1.0
    return {
        "metric": "ARC residual overhead: (fused ARC quantize + NVFP4 GEMM over K+S) / (same with S=0, GEMM over K) - 1",
        "value": round(overhead, 4), "unit": "fraction", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": False, "data": "synthetic", "impl": "ours",
        "config": {"workload": "arc_gemm: activations 8192x4096 (256 outlier channels x30), "
                               "weights 4096x4096, NVFP4, tiled scales, bf16 output",
                   "batches_per_step": U, "input_sets": R},
        "kernels_us": {k: round(v, 3) for k, v in us.items()},
        "gemm_tflops": {k: round(v, 1) for k, v in tf.items()},
        "roofline": {"bound": "tensor", "kernel": "gemm_K4352", "achieved": round(tf["gemm_K4352"], 1),
                     "peak": round(fp4_peak / 1e12, 1), "unit": "TFLOP/s",
                     "frac": round(tf["gemm_K4352"] * 1e12 / fp4_peak, 4),
                     "peak_source": f"{src} bf16 x 4 (nominal dense FP4 : bf16 ratio)"},
        "pages_overhead": "about 4.9% of total latency (ARCQuant, Resultats Experimentaux, Efficacite)",
        "clocks": clocks,
    }


def cpu_baseline(wl, x_np, raw, budget_s: float = 20.0):
    """The oracle as it stands, single-threaded on the host, on a bounded sample
    of the same workload (whole rows); GB/s of bf16 input."""
    import oracle
    name = wl["name"]
    M, K = wl["M"], wl["K"]

    def run(rows):
        xb = x_np[rows]
        if name == "mxfp4":
            c, s = oracle.quantize_mxfp4(xb)
            oracle.dequantize_bf16("mxfp4", c, s)
        elif name == "nvfp4":
            oracle.quantize_nvfp4(xb)
        elif name.startswith("hadamard"):
            oracle.hadamard_quantize(xb, wl["had"], "nvfp4", s_t=0.01)
        elif name.startswith("arc"):
            _, gamma, perm, outl = raw
            oracle.arc(xb, gamma, perm, outl, s_t=0.01, fmt=wl["fmt"].lower())
        elif name == "dual":
            c, s, g, _ = oracle.hadamard_quantize(xb, 512, "dual")
            oracle.dequantize_bf16("dual", c, s, g, inv_had=512)

    # calibrate on a few rows, then size the sample to the budget
    r = 8
    t = time.perf_counter()
    run(np.arange(r))
    per_row = (time.perf_counter() - t) / r
    n = int(min(M, max(16, budget_s / max(per_row, 1e-9))))
    rows = np.arange(n)
    t = time.perf_counter()
    run(rows)
    dt = time.perf_counter() - t
    return {"value": round(n * K * 2 / dt / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {n} of {M} rows ({n * K} elements), {dt:.1f} s",
            "seconds": round(dt, 2), **host_info()}


def host_info() -> dict:
    """The host the oracle ran on: its logical CPU count and model name.  The
    oracle is single-threaded scalar C, so it used one of them."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model, "threads_used": 1}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    """The oracle (plain C, one core) timed as this metric's reference arm."""
    wl = make_workload(args.workload, args.rows)
    raw = wl["x"]()
    x_np = raw[0] if isinstance(raw, tuple) else raw
    import oracle
    M, K = wl["M"], wl["K"]
    steps, warm = args.steps, args.warmup
    # each step: a bounded row sample, sized so all steps take ~2 minutes at most
    probe = cpu_baseline(wl, x_np, raw, budget_s=0.5)
    per_row = probe["seconds"] / int(probe["sample"].split()[1])
    budget_per_step = 120.0 / max(1, steps + warm)
    n = int(min(M, max(1, budget_per_step / max(per_row, 1e-9))))
    rows = np.arange(n)

    def one():
        xb = x_np[rows]
        if wl["name"] == "mxfp4":
            c, s = oracle.quantize_mxfp4(xb)
            oracle.dequantize_bf16("mxfp4", c, s)
        elif wl["name"] == "nvfp4":
            oracle.quantize_nvfp4(xb)
        elif wl["name"].startswith("hadamard"):
            oracle.hadamard_quantize(xb, wl["had"], "nvfp4", s_t=0.01)
        elif wl["name"].startswith("arc"):
            _, gamma, perm, outl = raw
            oracle.arc(xb, gamma, perm, outl, s_t=0.01, fmt=wl["fmt"].lower())
        else:
            c, s, g, _ = oracle.hadamard_quantize(xb, 512, "dual")
            oracle.dequantize_bf16("dual", c, s, g, inv_had=512)

    for _ in range(warm):
        one()
    t = time.perf_counter()
    for _ in range(steps):
        one()
    dt = time.perf_counter() - t
    v = n * K * 2 * steps / dt / 1e9
    return {
        "metric": METRIC, "value": round(v, 6), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": warm, "ms_per_step": round(dt / steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl["desc"], "M": M, "K": K, "format": wl["fmt"],
                   "hadamard": wl["had"], "parallelism": f"dp{world}"},
        "impl": "reference",
        "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"first {n} of {M} rows per step", **host_info()},
        "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dual",
                    help="dual (default) | mxfp4 | nvfp4 | hadamard128 | hadamard16 | hadamard32 | arc | "
                         "arc_mxfp4 | arc_int4 | arc_gemm")
    ap.add_argument("--rows", type=int, default=0,
                    help="override the workload's row count (small cases for profiler captures)")
    ap.add_argument("--units", type=int, default=0,
                    help="batches per step (default: about 24 GB of algorithmic traffic per step)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every call of the timed phases through the C ABI instead of "
                         "replaying a CUDA graph of them")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
    if args.workload == "arc_gemm":
        if rank == 0:
            print(json.dumps(run_arc_gemm(args, local_rank)), flush=True)
        return
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.barrier()
            tdist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
