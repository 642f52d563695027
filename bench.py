#!/usr/bin/env python
"""Benchmark of the grouped 4-bit MoE expert path on B200.

One step = one pass of the whole path over one batch of synthetic tokens:
route_permute -> projection 1 (gate_up) -> projection 2 (down) -> combine.
Decode workloads (T <= 8 tokens) run the grouped GEMV; prefill workloads the
tcgen05 grouped GEMM.  The activation between the projections (a GLU) is not
part of the path: projection 2 reads a resident synthetic [T*k, K2] input.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl libgnf4|reference]

Prints ONE JSON line (rank 0).  For N > 1 (torchrun) every rank runs its own
replica of the workload (no data-path collective; weak scaling) and the time
is the max over ranks.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_grouped_moe_b200 import inputs  # noqa: E402

METRIC = "grouped 4-bit GEMM TFLOP/s (prefill) & weight GB/s (decode) vs B200 roofline"
DEFAULT_WORKLOAD = "kimi-prefill"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
N_WEIGHT_COPIES = 4  # rotating copies when one weight stack fits in L2 (--weight-copies overrides)
L2_BYTES = 126 * 2**20
N_BATCHES = 8
GRAPH_STEPS = 20  # steps captured per CUDA graph (decode timing only)
DOMINANT_REPS = 60  # launches of the dominant kernel timed one by one (median, p10, p90)
# Nominal dense peaks of one B200 (context beside the measured ones): TFLOP/s per MMA kind, HBM3e GB/s.
NOMINAL = {"bf16": 2250.0, "fp8": 4500.0, "fp4": 9000.0, "hbm_gbs": 7700.0}


# ------------------------------------------------------------------ helpers


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "bit_grouped_moe_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel_key, sha):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it stands now."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel_key)
    if not e or e.get("source_sha") != sha:
        return None
    return e.get("dram_bytes_per_launch_full_size")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled in the background."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, uuid: str | None = None):
        self.index = index
        self.uuid = uuid
        self.samples = []
        self.proc = None
        self.thread = None
        self.ident = None

    def gpu_id(self) -> str:
        """The GPU for nvidia-smi: by UUID, which names the device this process
        computes on whatever CUDA_VISIBLE_DEVICES remaps; by index when
        nvidia-smi does not know that UUID."""
        if self.uuid:
            ident = self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid
            try:
                r = subprocess.run(["nvidia-smi", "-i", ident, "--query-gpu=uuid", "--format=csv,noheader"],
                                   capture_output=True, text=True, timeout=20)
                if r.returncode == 0 and r.stdout.strip():
                    return ident
            except (OSError, subprocess.TimeoutExpired):
                pass
        return str(self.index)

    def start(self):
        self.ident = self.gpu_id()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 - 0.15 <= t <= t1 + 0.15]
        if not rows and self.samples:
            rows = [min(self.samples, key=lambda ts: min(abs(ts[0] - t0), abs(ts[0] - t1)))[1]]
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 8:
                continue
            try:
                mhz.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz), "gpu": self.ident}


def gpu_uuid(local: int) -> str | None:
    """UUID of the CUDA device `local` as torch sees it (None if unavailable)."""
    try:
        import torch

        u = getattr(torch.cuda.get_device_properties(local), "uuid", None)
        return str(u) if u else None
    except Exception:  # noqa: BLE001 -- clocks then fall back to the index
        return None


# ------------------------------------------------------------------ workload


class Workload:
    """Device-resident inputs of one workload: rotating weight copies larger
    than L2, a set of token batches, and the step's output buffers."""

    def __init__(self, name, device, seed, build_host_copy, swiglu=False, dgrad=False, w4a8=False,
                 fused_combine=False, w4a8x2=False, w4a4=False, native=True):
        import torch

        from bit_grouped_moe_b200 import gnf4

        self.g = gnf4
        self.torch = torch
        self.wl = inputs.WORKLOADS[name]
        wl = self.wl
        self.name = name
        self.dev = device
        self.T, self.k, self.E = wl.T, wl.k, wl.E
        self.M = self.T * self.k
        self.decode = self.T <= gnf4.MAX_GEMV_ROWS
        self.p1, self.p2 = wl.projections[0], wl.projections[-1]
        rng = inputs.rng(seed)
        # token batches (ids, router weights, x) resident on the device; host copies kept for e2e
        self.batches = []
        for _ in range(N_BATCHES):
            ids, wts = inputs.routing_for(wl, rng)
            x = inputs.bf16_normal(rng, (self.T, self.p1.K))
            self.batches.append((ids, wts, x))
        self.d_batches = [(torch.from_numpy(i).to(device), torch.from_numpy(w).to(device),
                           torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device))
                          for (i, w, x) in self.batches]
        # weight stacks: N_WEIGHT_COPIES rotating copies of both projections
        self.host_stacks = None
        self.stacks = []
        for c in range(N_WEIGHT_COPIES):
            st = []
            for j, p in enumerate((self.p1, self.p2)):
                st.append(self._stack(wl.fmt, p, seed * 100 + c * 10 + j, keep_host=(c == 0 and build_host_copy)))
            self.stacks.append(st)
        self.h = torch.from_numpy(inputs.bf16_normal(rng, (self.M, self.p2.K)).view(np.int16)).view(
            torch.bfloat16).to(device)
        # outputs and scratch
        E, M = self.E, self.M
        self.off = torch.empty(E + 1, dtype=torch.int32, device=device)
        self.s2f = torch.empty(M, dtype=torch.int32, device=device)
        self.f2s = torch.empty(M, dtype=torch.int32, device=device)
        self.xs = torch.empty(M, self.p1.K, dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(max(gnf4.route_workspace_bytes(self.T, self.k, E), 16), dtype=torch.uint8,
                              device=device)
        self.y1 = torch.empty(M, self.p1.N, dtype=torch.bfloat16, device=device)
        self.y2 = torch.empty(M, self.p2.N, dtype=torch.bfloat16, device=device)
        self.out = torch.empty(self.T, self.p2.N, dtype=torch.bfloat16, device=device)
        # host routing of every batch: number of experts hit (algorithmic bytes)
        self.hit = [int(np.count_nonzero(np.bincount(b[0].reshape(-1), minlength=E))) for b in self.batches]
        f = gnf4
        self.fn = {("nf4", True): f.grouped_gemv_nf4, ("nf4", False): f.grouped_gemm_nf4,
                   ("mxfp4", True): f.grouped_gemv_mxfp4, ("mxfp4", False): f.grouped_gemm_mxfp4}[
            (wl.fmt, self.decode)]
        # optional backward step: the data gradients of both projections
        self.dgrad = dgrad
        if dgrad:
            self.decode = False  # the dgrad call has no decode variant
            self.dy1 = torch.from_numpy(inputs.bf16_normal(rng, (M, self.p1.N)).view(np.int16)).view(
                torch.bfloat16).to(device)
            self.dy2 = torch.from_numpy(inputs.bf16_normal(rng, (M, self.p2.N)).view(np.int16)).view(
                torch.bfloat16).to(device)
            self.dx1 = torch.empty(M, self.p1.K, dtype=torch.bfloat16, device=device)
            self.dh = torch.empty(M, self.p2.K, dtype=torch.bfloat16, device=device)
            self.dfn = f.grouped_dgrad_nf4 if wl.fmt == "nf4" else f.grouped_dgrad_mxfp4
        # optional native W4A8 mode (MXFP4 stacks): both projections' activations are
        # quantised to MXFP8 every step and the block-scaled GEMM runs on the codes
        self.w4a8 = w4a8 or w4a8x2 or w4a4
        self.split = w4a8x2  # two-term activations (hi + lo): the bf16-activation accuracy on the native path
        self.a4 = w4a4       # MXFP4 activations (kind::mxf4)
        if self.w4a8:
            assert wl.fmt == "mxfp4", "the W4A8 mode runs on MXFP4 weight stacks"
            self.decode = False  # one GEMM path for every group size
            cw = 2 if w4a4 else 1  # activation codes per byte
            self.qa1 = torch.empty(M, self.p1.K // cw, dtype=torch.uint8, device=device)
            self.sa1 = torch.empty(M, self.p1.K // 32, dtype=torch.uint8, device=device)
            self.qa2 = torch.empty(M, self.p2.K // cw, dtype=torch.uint8, device=device)
            self.sa2 = torch.empty(M, self.p2.K // 32, dtype=torch.uint8, device=device)
            if self.split:
                self.la1 = torch.empty_like(self.qa1)
                self.ls1 = torch.empty_like(self.sa1)
                self.la2 = torch.empty_like(self.qa2)
                self.ls2 = torch.empty_like(self.sa2)
        # the second projection's GEMV (decode) or GEMM (prefill, every group decoded) carries the top-k combine
        self.fused_combine = fused_combine and not dgrad and not self.w4a8
        if self.fused_combine:
            self.fn2c = ({"nf4": f.grouped_gemv_nf4_combine, "mxfp4": f.grouped_gemv_mxfp4_combine} if self.decode else
                         {"nf4": f.grouped_gemm_nf4_combine, "mxfp4": f.grouped_gemm_mxfp4_combine})[wl.fmt]
            self.cnt = torch.zeros(max(f.combine_counters_bytes(self.T, self.p2.N) // 4, 1), dtype=torch.int32,
                                   device=device)
        # optional fused gate_up + SwiGLU first projection: h [M, N1/2] feeds the second
        self.swiglu = swiglu
        if swiglu:
            assert self.p1.N // 2 == self.p2.K, "SwiGLU needs the second projection's K = first projection's N / 2"
            self.fn1 = {("nf4", True): f.grouped_gemv_nf4_swiglu, ("nf4", False): f.grouped_gemm_nf4_swiglu,
                        ("mxfp4", True): f.grouped_gemv_mxfp4_swiglu, ("mxfp4", False): f.grouped_gemm_mxfp4_swiglu}[
                (wl.fmt, self.decode)]
            self.hs = torch.empty(M, self.p1.N // 2, dtype=torch.bfloat16, device=device)
        # MXFP4 prefill: groups of at most 96 rows on the native two-term path (the
        # GEMM call with a workspace), larger groups on the decode path
        ws_n = [gnf4.mxfp4_workspace_bytes(M, p.K) for p in (self.p1, self.p2)]
        self.native = (native and wl.fmt == "mxfp4" and not self.decode and not dgrad and not self.w4a8
                       and not swiglu and min(ws_n) > 0)
        if self.native:
            self.mws = torch.empty(max(ws_n), dtype=torch.uint8, device=device)  # the projections run in turn
            self.fn = lambda a, w, s, y, offsets: gnf4.grouped_gemm_mxfp4_ws(a, w, s, y, self.mws, offsets=offsets)
        lim = gnf4.mxfp4_native_max_rows()
        self.native_rows = []  # rows in groups the native path takes, per batch
        for b in self.batches:
            sizes = np.bincount(b[0].reshape(-1), minlength=E)
            self.native_rows.append(int(sizes[sizes <= lim].sum()) if self.native else 0)

    def _stack(self, fmt, p, seed, keep_host):
        torch = self.torch
        E = self.E
        if keep_host:  # the copy the CPU baseline also reads is drawn on the host
            rng = inputs.rng(seed)
            if fmt == "nf4":
                w, s = inputs.nf4_direct(rng, E, p.N, p.K)
            else:
                w, s = inputs.mxfp4_random(rng, E, p.N, p.K)
            if self.host_stacks is None:
                self.host_stacks = []
            self.host_stacks.append((w, s))
            return torch.from_numpy(w).to(self.dev), torch.from_numpy(s).to(self.dev)
        w = inputs.device_random_bytes(seed, (E, p.N, p.K // 2), device=self.dev)
        if fmt == "nf4":
            s = inputs.device_absmax(seed + 1, (E, p.N, p.K // 64), device=self.dev)
        else:
            s = inputs.device_random_bytes(seed + 1, (E, p.N, p.K // 32), device=self.dev, lo=118, hi=131)
        return w, s

    # bytes / flops -----------------------------------------------------
    def weight_bytes(self, p, hit):
        per_elem_scale = 4 / 64 if self.wl.fmt == "nf4" else 1 / 32
        return int(hit * p.N * (p.K // 2 + p.K * per_elem_scale))

    def proj_bytes(self, p, hit):
        """Algorithmic bytes of one projection launch: weights + scales of the
        experts hit, activations read, outputs written (N/2 columns for the
        fused gate_up + SwiGLU first projection)."""
        n_out = p.N // 2 if (self.swiglu and p is self.p1) else p.N
        return self.weight_bytes(p, hit) + self.M * p.K * 2 + self.M * n_out * 2

    def step_weight_bytes(self, i):
        h = self.hit[i % N_BATCHES]
        return self.weight_bytes(self.p1, h) + self.weight_bytes(self.p2, h)

    def step_flops(self):
        return 2 * self.M * (self.p1.N * self.p1.K + self.p2.N * self.p2.K)

    # one step ------------------------------------------------------------
    def step(self, i, ev=None):
        g = self.g
        ids, wts, x = self.d_batches[i % N_BATCHES]
        (w1, s1), (w2, s2) = self.stacks[i % N_WEIGHT_COPIES]
        g.route_permute(ids, x, self.E, self.off, self.s2f, self.f2s, self.xs, self.ws)
        if self.dgrad:  # backward through both projections: dH = dY2 . W2, dX = dY1 . W1
            self.dfn(self.dy2, w2, s2, self.dh, offsets=self.off)
            if ev is not None:
                ev[0].record()
            self.dfn(self.dy1, w1, s1, self.dx1, offsets=self.off)
            if ev is not None:
                ev[1].record()
            return
        if self.w4a8:
            self._quant1()
        if ev is not None:
            ev[0].record()
        self.project(w1, s1, w2, s2, ev, wts=wts)
        if not self.fused_combine:
            g.combine(self.y2, self.f2s, wts, self.out)

    def _quant1(self):
        if self.a4:
            self.g.quantize_mxfp4_act(self.xs, self.qa1, self.sa1)
        elif self.split:
            self.g.quantize_mxfp8_split(self.xs, self.qa1, self.sa1, self.la1, self.ls1)
        else:
            self.g.quantize_mxfp8(self.xs, self.qa1, self.sa1)

    def project(self, w1, s1, w2, s2, ev=None, quantize_first=False, wts=None):
        if self.w4a8:
            g = self.g
            if quantize_first:
                self._quant1()
            if self.a4:
                g.grouped_gemm_w4a4(self.qa1, self.sa1, w1, s1, self.y1, offsets=self.off)
            elif self.split:
                g.grouped_gemm_w4a8x2(self.qa1, self.sa1, self.la1, self.ls1, w1, s1, self.y1, offsets=self.off)
            else:
                g.grouped_gemm_w4a8(self.qa1, self.sa1, w1, s1, self.y1, offsets=self.off)
            if ev is not None:
                ev[1].record()
            if self.a4:
                g.quantize_mxfp4_act(self.h, self.qa2, self.sa2)
                g.grouped_gemm_w4a4(self.qa2, self.sa2, w2, s2, self.y2, offsets=self.off)
            elif self.split:
                g.quantize_mxfp8_split(self.h, self.qa2, self.sa2, self.la2, self.ls2)
                g.grouped_gemm_w4a8x2(self.qa2, self.sa2, self.la2, self.ls2, w2, s2, self.y2, offsets=self.off)
            else:
                g.quantize_mxfp8(self.h, self.qa2, self.sa2)
                g.grouped_gemm_w4a8(self.qa2, self.sa2, w2, s2, self.y2, offsets=self.off)
            return
        if self.swiglu:
            self.fn1(self.xs, w1, s1, self.hs, offsets=self.off)
        else:
            self.fn(self.xs, w1, s1, self.y1, offsets=self.off)
        if ev is not None:
            ev[1].record()
        a2 = self.hs if self.swiglu else self.h
        if self.fused_combine:
            self.fn2c(a2, w2, s2, self.y2, self.s2f, self.f2s, wts, self.out, self.cnt, offsets=self.off)
        else:
            self.fn(a2, w2, s2, self.y2, offsets=self.off)

    def dominant(self, i):
        """Launches the dominant kernel alone (the first projection, or dX of
        it for the backward step) on weight copy i, with the routing of the
        last step: the kernel the roofline is reported for."""
        (w1, s1), _ = self.stacks[i % N_WEIGHT_COPIES]
        g = self.g
        if self.dgrad:
            self.dfn(self.dy1, w1, s1, self.dx1, offsets=self.off)
        elif self.w4a8:
            if self.a4:
                g.grouped_gemm_w4a4(self.qa1, self.sa1, w1, s1, self.y1, offsets=self.off)
            elif self.split:
                g.grouped_gemm_w4a8x2(self.qa1, self.sa1, self.la1, self.ls1, w1, s1, self.y1, offsets=self.off)
            else:
                g.grouped_gemm_w4a8(self.qa1, self.sa1, w1, s1, self.y1, offsets=self.off)
        elif self.swiglu:
            self.fn1(self.xs, w1, s1, self.hs, offsets=self.off)
        else:
            self.fn(self.xs, w1, s1, self.y1, offsets=self.off)

    def launches_per_step(self):
        # route (one launch for at most 256 pairs, else hist + scan + scatter + gather) + 2 projections + combine
        route = 1 if 0 < self.M <= 256 else 4
        combine = 0 if (self.dgrad or self.fused_combine) else 1
        # the native MXFP4 call: split quantiser + native GEMM + decode GEMM per projection (M > 96); the
        # fused-combine second projection is one launch
        native = (2 if self.fused_combine else 4) if self.native else 0
        return route + 2 + combine + (2 if self.w4a8 else 0) + native


# ------------------------------------------------------------------ distributed


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def engagement(g) -> dict:
    """libgnf4's engagement counters for the entry points called since the
    last reset: calls, calls that enqueued work, and how many reached each
    kernel family (decode-path tcgen05, native block-scaled, GEMV).  Host-side
    counters; reading them touches no device."""
    out = {}
    for name in g.call_stats_names():
        st = g.call_stats_get(name)
        if st["calls"]:
            out[name[len("gnf4_"):]] = {k: v for k, v in st.items() if v or k == "calls"}
    return out


def max_over_ranks(value: float, world: int) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------ CPU (oracle) legs


def oracle_step(wl_obj, batch_i, n_slice=None):
    """The same step computed by the oracle on the host (fp64): route, gather,
    both projections (optionally on their first n_slice weight rows) and the
    combine.  Returns (weight bytes, flops) of the work done."""
    import torch

    import oracle

    ids, wts, x = wl_obj.batches[batch_i % N_BATCHES]
    E, k = wl_obj.E, wl_obj.k
    off, s2f, f2s, _ = oracle.route(ids, E)
    xs = oracle.gather(x, k, s2f, int(off[E]))
    (w1, s1), (w2, s2) = wl_obj.host_stacks
    n1 = wl_obj.p1.N if n_slice is None else min(n_slice, wl_obj.p1.N)
    n2 = wl_obj.p2.N if n_slice is None else min(n_slice, wl_obj.p2.N)
    if getattr(wl_obj, "a4", False):
        def gemm(a_bits, w, s, off):
            return oracle.grouped_gemm_w4a4(*oracle.quant_mxfp4_act(a_bits), w, s, off)
    elif getattr(wl_obj, "split", False):
        def gemm(a_bits, w, s, off):
            return oracle.grouped_gemm_w4a8x2(*oracle.quant_mxfp8_split(a_bits), w, s, off)
    elif getattr(wl_obj, "w4a8", False):
        def gemm(a_bits, w, s, off):
            qa, sa = oracle.quant_mxfp8(a_bits)
            return oracle.grouped_gemm_w4a8(qa, sa, w, s, off)
    else:
        gemm = oracle.grouped_gemm_nf4 if wl_obj.wl.fmt == "nf4" else oracle.grouped_gemm_mxfp4
    gemm(xs, np.ascontiguousarray(w1[:, :n1]), np.ascontiguousarray(s1[:, :n1]), off)
    y2 = gemm(wl_obj.h_host, np.ascontiguousarray(w2[:, :n2]), np.ascontiguousarray(s2[:, :n2]), off)
    y2_bits = np.zeros((wl_obj.M, n2), np.uint16)
    y2_bits[:y2.shape[0]] = torch.from_numpy(y2).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    oracle.combine(y2_bits, f2s, wts)
    hit = wl_obj.hit[batch_i % N_BATCHES]
    scale = 4 / 64 if wl_obj.wl.fmt == "nf4" else 1 / 32
    wbytes = hit * (n1 * wl_obj.p1.K + n2 * wl_obj.p2.K) * (0.5 + scale)
    return int(wbytes), 2 * wl_obj.M * (n1 * wl_obj.p1.K + n2 * wl_obj.p2.K)


def cpu_baseline(wl_obj, budget_s=15.0, threads=None):
    """Oracle timed on the host cores (all of them, or `threads`) on a bounded
    sample of the workload."""
    import oracle

    cores = threads or os.cpu_count() or 1
    oracle.set_threads(cores)
    # calibrate the weight-row slice so that one step costs ~budget/6
    t0 = time.perf_counter()
    oracle_step(wl_obj, 0, n_slice=64)
    t_unit = max(time.perf_counter() - t0, 1e-3)
    n_slice = int(min(max(64, 64 * (budget_s / 6) / t_unit), max(wl_obj.p1.N, wl_obj.p2.N)))
    n_slice -= n_slice % 8
    tot_b, tot_f, steps = 0, 0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and steps < 400:
        b, f = oracle_step(wl_obj, steps, n_slice=n_slice)
        tot_b += b
        tot_f += f
        steps += 1
    dt = time.perf_counter() - t0
    return {"bytes": tot_b, "flops": tot_f, "seconds": dt, "cores": cores, "steps": steps, "n_slice": n_slice}


def roofline(wl, args, peaks, peak_src, dom_ms, hit, dom_stats, traffic):
    """Roofline of the dominant kernel (median of its own timed loop).

    F = 2*M*N*K useful flops; B = algorithmic bytes (weights + scales of the
    experts hit, activations read once, output written once).  The bound is
    the combined one, t = max(F / tensor peak, B / HBM peak), with the tensor
    peak of the MMA kind the kernel executes expressed in useful flops (the
    two-term form issues two fp8-rate MMAs per useful one).  `frac` = t /
    measured time against the measured peaks; the same against the nominal
    dense peaks is `frac_nominal`.  The measured tensor peak is the burst
    figure, or the sustained one when the kernel's own loop ran power-capped
    (sw_power_cap active or the median SM clock below 90% of max)."""
    p = wl.p1
    M, N, K = wl.M, p.N, p.K
    F = 2.0 * M * N * K
    wbytes = wl.weight_bytes(p, hit)
    if wl.dgrad:
        io = 2 * M * N + 2 * M * K  # dY read, dX written
        kind, per = "bf16", 1.0
    elif wl.w4a8:
        if wl.a4:
            abytes, kind, per = M * K // 2 + M * K // 32, "fp4", 1.0
        elif wl.split:
            abytes, kind, per = 2 * (M * K + M * K // 32), "fp8", 0.5
        else:
            abytes, kind, per = M * K + M * K // 32, "fp8", 1.0
        io = abytes + 2 * M * N
    else:
        n_out = N // 2 if wl.swiglu else N
        io = 2 * M * K + 2 * M * n_out
        kind, per = "bf16", 1.0
        if wl.native:
            # the native path's rows: two e4m3 terms + scales written by the quantiser and read by the GEMM; its
            # MMAs run at the fp8 rate, two per useful product, so its useful-flop peak is the bf16 one
            io += 2 * 2 * wl.native_rows[0] * (K + K // 32)
    B = float(wbytes + io)
    ratio = {"bf16": 1.0, "fp8": 2.0, "fp4": 4.0}[kind]
    dc = dom_stats.get("clocks") or {}
    capped = ("sw_power_cap" in (dc.get("reasons") or [])) or (
        dc.get("sm_mhz") is not None and dc.get("sm_max_mhz") and dc["sm_mhz"] < 0.9 * dc["sm_max_mhz"])
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * ratio * per
    sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * ratio * per
    tpk = sust if capped else burst
    nominal_t = NOMINAL[kind] * per
    hbm = peaks["hbm_gbs"]
    t = dom_ms / 1e3
    t_tensor, t_hbm = F / (tpk * 1e12), B / (hbm * 1e9)
    bound = "tensor" if t_tensor >= t_hbm else "hbm"
    t_nom = max(F / (nominal_t * 1e12), B / (NOMINAL["hbm_gbs"] * 1e9))
    achieved = F / t / 1e12 if bound == "tensor" else B / t / 1e9
    kname = (f"gnf4_grouped_gemm_mxfp4_ws ({p.name}, K={K}, N={N}): quant_mxfp8_rows_kernel + "
             f"gemm_mx_kernel<two-term> on the {wl.native_rows[0]} rows of groups <= 96 rows, "
             f"gemm_tc_kernel<mxfp4> on the rest (3 launches)" if wl.native else
             f"dgrad_tc_kernel<{wl.wl.fmt}> (dX of {p.name}, K={K}, N={N})" if wl.dgrad else
             f"gemm_mx_kernel<W4A4> ({p.name}, K={K}, N={N})" if wl.a4 else
             f"gemm_mx_kernel<two-term> ({p.name}, K={K}, N={N})" if wl.split else
             f"gemm_mx_kernel<W4A8> ({p.name}, K={K}, N={N})" if wl.w4a8 else
             f"gemv_kernel<{wl.wl.fmt}{', swiglu' if wl.swiglu else ''}> ({p.name}, K={K}, N={N})" if wl.decode else
             f"gemm_tc_kernel<{wl.wl.fmt}{', swiglu' if wl.swiglu else ''}> ({p.name}, K={K}, N={N})")
    return {
        "bound": bound, "achieved": round(achieved, 1), "peak": round(tpk if bound == "tensor" else hbm, 1),
        "unit": "TFLOP/s" if bound == "tensor" else "GB/s", "frac": round(max(t_tensor, t_hbm) / t, 4),
        "traffic": traffic, "kernel": kname,
        "algorithmic_flops_per_launch": int(F), "algorithmic_bytes_per_launch": int(B),
        "experts_hit": int(hit), "launch_us": dom_stats,
        "tensor": {"achieved_tflops": round(F / t / 1e12, 1), "mma_kind": kind,
                   "peak_measured": round(tpk, 1), "frac_measured": round(F / t / 1e12 / tpk, 4),
                   "peak_nominal": round(nominal_t, 1), "frac_nominal": round(F / t / 1e12 / nominal_t, 4),
                   "peak_burst": round(burst, 1), "peak_sustained": round(sust, 1),
                   "peak_choice": "sustained (loop ran power-capped)" if capped else "burst"},
        "hbm": {"achieved_gbs": round(B / t / 1e9, 1), "peak_measured": hbm,
                "frac_measured": round(B / t / 1e9 / hbm, 4), "peak_nominal": NOMINAL["hbm_gbs"],
                "frac_nominal": round(B / t / 1e9 / NOMINAL["hbm_gbs"], 4)},
        "combined_bound_us": round(max(t_tensor, t_hbm) * 1e6, 3), "frac_nominal": round(t_nom / t, 4),
        "peak_source": f"{peak_src} (MEASURED_PEAKS.json: bf16_tflops / bf16_tflops_sustained x the nominal "
                       f"{kind}/bf16 ratio {ratio:g}{', halved for the two-term form' if per != 1 else ''}; hbm_gbs)",
        **({"tensor_note": "native rows run kind::mxf8f6f4 at 2x the bf16 rate with two MMAs per useful product, "
                           "the rest kind::f16: both at the bf16 useful-flop peak"} if wl.native else {}),
    }



# ------------------------------------------------------------------ main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="libgnf4", choices=["libgnf4", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dgrad", action="store_true",
                    help="time the backward step instead: route + the dgrad of both projections (TFLOP/s)")
    ap.add_argument("--no-graph", action="store_true",
                    help=f"decode: skip timing the steps replayed from one CUDA graph of {GRAPH_STEPS} steps")
    ap.add_argument("--w4a8", action="store_true",
                    help="MXFP4 workloads: native W4A8 mode (MXFP8 activations, block-scaled tcgen05 GEMM)")
    ap.add_argument("--w4a8x2", action="store_true",
                    help="MXFP4 workloads: two-term native mode (hi + lo MXFP8 activations, the bf16-activation "
                         "accuracy on the block-scaled tcgen05 GEMM)")
    ap.add_argument("--w4a4", action="store_true",
                    help="MXFP4 workloads: native W4A4 mode (MXFP4 activations, kind::mxf4 block-scaled GEMM)")
    ap.add_argument("--fused-combine", action="store_true",
                    help="run the top-k combine inside the second projection's launch (decode: the GEMV epilogue; "
                         "prefill: after each GEMM unit, every group on the decode path) instead of as its own launch")
    ap.add_argument("--no-native", action="store_true",
                    help="MXFP4 prefill: every group on the decode path (gnf4_grouped_gemm_mxfp4 without a workspace)")
    ap.add_argument("--swiglu", action="store_true",
                    help="first projection = fused gate_up + SwiGLU (gate rows first); the second reads its output")
    ap.add_argument("--weight-copies", type=int, default=None,
                    help="rotating copies of every weight stack (4 keeps the rotation larger than L2)")
    args = ap.parse_args()
    wl0 = inputs.WORKLOADS[args.workload]
    if args.weight_copies is None:
        # one stack of the first projection larger than 3x L2 needs no rotation
        per = 0.5 + (4 / 64 if wl0.fmt == "nf4" else 1 / 32)
        one = wl0.E * wl0.projections[0].N * wl0.projections[0].K * per
        args.weight_copies = 1 if one > 3 * L2_BYTES else N_WEIGHT_COPIES
    globals()["N_WEIGHT_COPIES"] = max(1, args.weight_copies)

    wl_def = inputs.WORKLOADS[args.workload]
    decode = wl_def.T <= 8 and not args.dgrad and not args.w4a8 and not args.w4a8x2 and not args.w4a4
    steps = args.steps if args.steps is not None else (20000 if decode else 200)
    warmup = args.warmup if args.warmup is not None else (100 if decode else 10)
    warmup = max(warmup, 3)

    world, rank, local = (1, 0, 0)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        return run_reference(args, steps, warmup, world)
    world, rank, local = dist_setup(args.gpus)
    return run_gpu(args, steps, warmup, world, rank, local, decode)


def _unit(decode):
    return ("GB/s", "weight GB/s") if decode else ("TFLOP/s", "TFLOP/s")


def _config(wl_obj_or_def, world):
    wl = wl_obj_or_def
    return {
        "workload": f"{wl.name}: {wl.fmt.upper()} grouped MoE experts, E={wl.E}, top-{wl.k}, T={wl.T} tokens",
        "experts": wl.E, "top_k": wl.k, "tokens_per_step": wl.T,
        "projections": [{"name": p.name, "K": p.K, "N": p.N} for p in wl.projections],
        "format": wl.fmt,
        "l2": (f"{N_WEIGHT_COPIES} rotating copies of every weight stack (inputs larger than L2)" if N_WEIGHT_COPIES > 1
               else "one copy of every weight stack: a stack alone is larger than L2") + f", {N_BATCHES} token batches",
        "parallelism": f"{world} independent replica(s)",
    }


def run_gpu(args, steps, warmup, world, rank, local, decode):
    import torch

    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    wl = Workload(args.workload, dev, seed=1234 + rank, build_host_copy=(rank == 0 and world == 1),
                  swiglu=args.swiglu, dgrad=args.dgrad, w4a8=args.w4a8, fused_combine=args.fused_combine,
                  w4a8x2=args.w4a8x2, w4a4=args.w4a4, native=not args.no_native)
    decode = wl.decode
    wl.h_host = wl.h.cpu().view(torch.int16).numpy().view(np.uint16)
    stream = torch.cuda.current_stream()

    # warm-up
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()
    assert wl.g.device_errors() == 0, "device error word set during warm-up"

    # timed region (inputs resident): K whole steps, no event inside it, so
    # consecutive launches keep their programmatic overlap
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local, gpu_uuid(local))
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    wl.g.call_stats_get(None, reset=True)  # count the timed steps' calls only
    t_wall0 = time.time()
    start.record(stream)
    for i in range(steps):
        wl.step(i)
    stop.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    engaged = engagement(wl.g)
    barrier(world)
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    ms_local = start.elapsed_time(stop)
    ms = max_over_ranks(ms_local, world)

    # the dominant kernel in a loop of its own: DOMINANT_REPS launches, each
    # bracketed by events on the launching stream, weight copies rotating (the
    # rotation is larger than L2 for the decode shapes; a prefill stack alone
    # is), routing of batch 0
    wl.step(0)
    torch.cuda.synchronize()
    dsampler = ClockSampler(local, gpu_uuid(local))
    dsampler.start()
    time.sleep(0.3)
    dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(DOMINANT_REPS)]
    torch.cuda.synchronize()
    d_wall0 = time.time()
    # a head start for the GPU (torch's spin kernel, ~2.5 ms): every launch of the
    # loop is queued before it runs, so the event pairs time the device only and
    # not the host's enqueue of a short kernel
    torch.cuda._sleep(5_000_000)
    for r, (a, b) in enumerate(dev_ev):
        a.record(stream)
        wl.dominant(r)
        b.record(stream)
    torch.cuda.synchronize()
    d_wall1 = time.time()
    time.sleep(0.2)
    dsampler.stop()
    dclocks = dsampler.summary(d_wall0, d_wall1)
    dom = sorted(a.elapsed_time(b) for a, b in dev_ev)
    dom_ms = statistics.median(dom)
    dom_stats = {"reps": len(dom), "median_us": round(dom_ms * 1e3, 3),
                 "p10_us": round(dom[int(0.1 * (len(dom) - 1))] * 1e3, 3),
                 "p90_us": round(dom[int(0.9 * (len(dom) - 1))] * 1e3, 3),
                 "mean_us": round(statistics.fmean(dom) * 1e3, 3), "clocks": dclocks}
    dom_hit = wl.hit[0]
    # host cost of one call (argument checks, tensor-map encodes, launch) through
    # the Python binding: enqueue time of the same launches, no events, no sync
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    for r in range(DOMINANT_REPS):
        wl.dominant(r)
    h1 = time.perf_counter()
    torch.cuda.synchronize()
    dom_stats["host_enqueue_us_per_call"] = round((h1 - h0) / DOMINANT_REPS * 1e6, 2)
    assert wl.g.device_errors() == 0, "device error word set during the timed steps"

    # e2e through the public API with host buffers (pinned), copies in the timed region.
    # Each batch's inputs (ids, router weights, x) are packed in one pinned
    # buffer, so a step makes one host->device copy and one device->host copy.
    def _pad16(n):
        return (n + 15) // 16 * 16

    ex = wl.batches[0]
    seg = [_pad16(ex[0].nbytes), _pad16(ex[1].nbytes), _pad16(ex[2].nbytes)]
    host_in = []
    for (ids, wts, x) in wl.batches:
        hb = torch.zeros(sum(seg), dtype=torch.uint8).pin_memory()
        o = 0
        for arr, n in zip((ids, wts, x), seg):
            hb[o:o + arr.nbytes] = torch.from_numpy(np.ascontiguousarray(arr).view(np.uint8).reshape(-1))
            o += n
        host_in.append(hb)
    d_in = torch.empty(sum(seg), dtype=torch.uint8, device=dev)
    d_ids = d_in[0:ex[0].nbytes].view(torch.int32).view(ex[0].shape)
    d_w = d_in[seg[0]:seg[0] + ex[1].nbytes].view(torch.float32).view(ex[1].shape)
    d_x = d_in[seg[0] + seg[1]:seg[0] + seg[1] + ex[2].nbytes].view(torch.bfloat16).view(ex[2].shape)
    out_dev = wl.dx1 if wl.dgrad else wl.out
    host_out = torch.empty(tuple(out_dev.shape), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(steps, 2000 if decode else steps))

    def e2e_step(i):
        d_in.copy_(host_in[i % N_BATCHES], non_blocking=True)
        (w1, s1), (w2, s2) = wl.stacks[i % N_WEIGHT_COPIES]
        g = wl.g
        g.route_permute(d_ids, d_x, wl.E, wl.off, wl.s2f, wl.f2s, wl.xs, wl.ws)
        if wl.dgrad:
            wl.dfn(wl.dy2, w2, s2, wl.dh, offsets=wl.off)
            wl.dfn(wl.dy1, w1, s1, wl.dx1, offsets=wl.off)
        else:
            wl.project(w1, s1, w2, s2, quantize_first=True, wts=d_w)
            if not wl.fused_combine:
                g.combine(wl.y2, wl.f2s, d_w, wl.out)
        host_out.copy_(out_dev, non_blocking=True)

    # Prefill: the steps are pipelined across three streams with double-buffered
    # inputs and outputs, so step i+1's upload and step i-1's download overlap
    # step i's kernels (each step's own copies stay inside the timed region).
    # Decode keeps one stream: its copies are a few KB, and the event waits of
    # the pipelined form cost what the overlap saved (measured).
    pipelined = not decode and not wl.fused_combine
    if pipelined:
        d_in2 = [d_in, torch.empty_like(d_in)]
        views = [(b[0:ex[0].nbytes].view(torch.int32).view(ex[0].shape),
                  b[seg[0]:seg[0] + ex[1].nbytes].view(torch.float32).view(ex[1].shape),
                  b[seg[0] + seg[1]:seg[0] + seg[1] + ex[2].nbytes].view(torch.bfloat16).view(ex[2].shape))
                 for b in d_in2]
        outs = [out_dev, torch.empty_like(out_dev)]
        host_outs = [host_out, torch.empty_like(host_out).pin_memory()]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        ev_in, ev_done, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def e2e_pipelined(i0, n):
            start = torch.cuda.Event()
            start.record(stream)
            s_in.wait_event(start)
            s_out.wait_event(start)
            for i in range(i0, i0 + n):
                b = i % 2
                ids_b, w_b, x_b = views[b]
                with torch.cuda.stream(s_in):
                    if i - i0 >= 2:
                        s_in.wait_event(ev_done[b])  # step i-2 has finished with this input buffer
                    d_in2[b].copy_(host_in[i % N_BATCHES], non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i - i0 >= 2:
                    stream.wait_event(ev_out[b])  # step i-2's output has been read back
                (w1, s1), (w2, s2) = wl.stacks[i % N_WEIGHT_COPIES]
                g = wl.g
                g.route_permute(ids_b, x_b, wl.E, wl.off, wl.s2f, wl.f2s, wl.xs, wl.ws)
                if wl.dgrad:
                    wl.dfn(wl.dy2, w2, s2, wl.dh, offsets=wl.off)
                    wl.dfn(wl.dy1, w1, s1, outs[b], offsets=wl.off)
                else:
                    wl.project(w1, s1, w2, s2, quantize_first=True, wts=w_b)
                    g.combine(wl.y2, wl.f2s, w_b, outs[b])
                ev_done[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[b])
                    host_outs[b].copy_(outs[b], non_blocking=True)
                    ev_out[b].record(s_out)
            for b in range(2):
                stream.wait_event(ev_out[b])
                stream.wait_event(ev_in[b])

    if pipelined:
        e2e_pipelined(0, warmup)
    else:
        for i in range(warmup):
            e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if pipelined:
        e2e_pipelined(0, e2e_steps)
    else:
        for i in range(e2e_steps):
            e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = int(sum(seg))  # one packed copy (ids, weights, x, each padded to 16 bytes)
    d2h = int(host_out.numel() * 2)

    # decode: the same steps replayed from one CUDA graph of GRAPH_STEPS steps
    graph = None
    if decode and not args.no_graph:
        gs = torch.cuda.Stream()
        gs.wait_stream(stream)
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gs):
            for i in range(2):
                wl.step(i)
            gs.synchronize()
            with torch.cuda.graph(cg, stream=gs):
                for i in range(GRAPH_STEPS):
                    wl.step(i)
        torch.cuda.synchronize()
        reps = max(1, steps // GRAPH_STEPS)
        for _ in range(3):
            cg.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(reps):
            cg.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        g_ms = max_over_ranks(g0.elapsed_time(g1), world) / (reps * GRAPH_STEPS)
        gbytes = sum(wl.step_weight_bytes(i) for i in range(GRAPH_STEPS)) / GRAPH_STEPS
        graph = {"ms_per_step": round(g_ms, 6), "value": round(world * gbytes / (g_ms / 1e3) / 1e9, 3),
                 "unit": "GB/s", "steps_per_graph": GRAPH_STEPS, "replays": reps}
        del cg
        assert wl.g.device_errors() == 0, "device error word set during the graph replays"

    unit, _ = _unit(decode)
    if decode:
        per_rank = sum(wl.step_weight_bytes(i) for i in range(steps))
        value = world * per_rank / (ms / 1e3) / 1e9
        e2e_val = world * sum(wl.step_weight_bytes(i) for i in range(e2e_steps)) / (e2e_ms / 1e3) / 1e9
    else:
        value = world * steps * wl.step_flops() / (ms / 1e3) / 1e12
        e2e_val = world * e2e_steps * wl.step_flops() / (e2e_ms / 1e3) / 1e12

    peaks, peak_src = load_peaks()
    kern_file = "gemv.cu" if decode else ("dgrad.cu" if wl.dgrad else ("mx.cu" if wl.w4a8 else "gemm_tc.cu"))
    kern_base = "gemm_mxfp4_ws" if wl.native else "gemv" if decode else ("dgrad_tc" if wl.dgrad else
                                       ("gemm_w4a4" if wl.a4 else ("gemm_w4a8x2" if wl.split else
                                                                  ("gemm_w4a8" if wl.w4a8 else "gemm_tc"))))
    kern_key = f"{kern_base}_{wl.wl.fmt}{'_swiglu' if wl.swiglu else ''}:{args.workload}:{wl.p1.name}"
    sha = kernel_source_sha(["mx.cu", "gemm_tc.cu", "common.cuh"] if wl.native else [kern_file, "common.cuh"])
    roof = roofline(wl, args, peaks, peak_src, dom_ms, dom_hit, dom_stats, committed_traffic(kern_key, sha))

    cpu = cpu1 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(wl)
        v = cb["bytes"] / cb["seconds"] / 1e9 if decode else cb["flops"] / cb["seconds"] / 1e12
        cpu = {"value": round(v, 6), "unit": unit, "cores": cb["cores"], "kind": "oracle",
               "sample": f"{cb['steps']} steps of the same workload on the first {cb['n_slice']} weight rows of "
                         f"each projection (route + fp64 grouped GEMM x2 + combine), {cb['seconds']:.1f} s"}
        c1 = cpu_baseline(wl, budget_s=8.0, threads=1)
        v1 = c1["bytes"] / c1["seconds"] / 1e9 if decode else c1["flops"] / c1["seconds"] / 1e12
        cpu1 = {"value": round(v1, 6), "unit": unit, "cores": 1, "kind": "oracle",
                "sample": f"{c1['steps']} steps on the first {c1['n_slice']} weight rows of each projection, "
                          f"{c1['seconds']:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": round(ms / steps, 6), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("e2m1 x e2m1 (fp32 accumulate)" if wl.a4 else
                      "(e4m3 hi + e4m3 lo) x e2m1 (fp32 accumulate)" if wl.split else
                      "e4m3 x e2m1 (fp32 accumulate)" if wl.w4a8 else "bf16"), "data": "synthetic",
            "config": dict(_config(wl.wl, world), **({"first_projection": "fused gate_up + SwiGLU"} if wl.swiglu else {}),
                           **({"activations": "MXFP4 (native W4A4 mode: quantised every step)"} if wl.a4 else
                              {"activations": "two-term MXFP8 hi + lo (quantised every step; bf16-activation accuracy)"}
                              if wl.split else
                              {"activations": "MXFP8 (native W4A8 mode: quantised every step)"} if wl.w4a8 else {}),
                           **({"combine": "in the second GEMV's epilogue" if wl.decode else
                                          "after each unit of the second GEMM (decode path for every group)"}
                              if wl.fused_combine else {}),
                           **({"mxfp4_path": "groups <= 96 rows: native two-term MXFP8 x e2m1 (kind::mxf8f6f4, "
                                             "bf16-activation accuracy); larger groups: decode to bf16 (kind::f16)"}
                              if wl.native else {}),
                           **({"step": "backward: route + dgrad of both projections"} if wl.dgrad else {})),
            "roofline": roof, "cpu_baseline": cpu, **({"cpu_baseline_1core": cpu1} if cpu1 else {}),
            "e2e": {"value": round(e2e_val, 3), "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps,
                    "copies": "overlapped with the neighbouring steps' kernels (copy streams, double buffers)"
                              if pipelined else "in stream order with the step's kernels"},
            "gpu_launches": steps * wl.launches_per_step(), "engagement": engaged, "clocks": clocks,
            "impl": "libgnf4", **({"cuda_graph": graph} if graph is not None else {}),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def run_reference(args, steps, warmup, world):
    """The oracle arm: the same metric computed by the CPU oracle on the box's
    host cores, each step a bounded sample of the workload."""
    import oracle

    wl_def = inputs.WORKLOADS[args.workload]
    decode = wl_def.T <= 8 and not args.w4a8 and not args.w4a8x2 and not args.w4a4
    unit, _ = _unit(decode)

    class HostWL:
        pass

    h = HostWL()
    h.wl = wl_def
    h.w4a8 = args.w4a8 or args.w4a8x2 or args.w4a4
    h.split = args.w4a8x2
    h.a4 = args.w4a4
    h.E, h.k, h.T = wl_def.E, wl_def.k, wl_def.T
    h.M = h.T * h.k
    h.p1, h.p2 = wl_def.projections[0], wl_def.projections[-1]
    rng = inputs.rng(1234)
    h.batches = []
    for _ in range(N_BATCHES):
        ids, wts = inputs.routing_for(wl_def, rng)
        x = inputs.bf16_normal(rng, (h.T, h.p1.K))
        h.batches.append((ids, wts, x))
    h.hit = [int(np.count_nonzero(np.bincount(b[0].reshape(-1), minlength=h.E))) for b in h.batches]
    # only the weight rows the sample touches are drawn
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    budget = 90.0 / (steps + warmup)
    n_slice = 64
    srng = inputs.rng(99)
    mk = inputs.nf4_direct if wl_def.fmt == "nf4" else inputs.mxfp4_random

    def stacks(ns):
        return [mk(srng, h.E, min(ns, p.N), p.K) for p in (h.p1, h.p2)]

    h.host_stacks = stacks(n_slice)
    h.h_host = inputs.bf16_normal(rng, (h.M, h.p2.K))
    t0 = time.perf_counter()
    oracle_step(h, 0, n_slice=n_slice)
    t1 = max(time.perf_counter() - t0, 1e-4)
    n_slice = int(max(8, min(max(h.p1.N, h.p2.N), n_slice * budget / t1)))
    n_slice -= n_slice % 8
    n_slice = max(n_slice, 8)
    h.host_stacks = stacks(n_slice)
    for i in range(warmup):
        oracle_step(h, i, n_slice=n_slice)
    tb, tf = 0, 0
    t0 = time.perf_counter()
    for i in range(steps):
        b, f = oracle_step(h, i, n_slice=n_slice)
        tb += b
        tf += f
    dt = time.perf_counter() - t0
    value = tb / dt / 1e9 if decode else tf / dt / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": round(dt * 1e3 / steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(_config(wl_def, world),
                       **({"activations": "MXFP4 (native W4A4 mode: quantised every step)"} if args.w4a4 else
                          {"activations": "two-term MXFP8 hi + lo (quantised every step; bf16-activation accuracy)"}
                          if args.w4a8x2 else
                          {"activations": "MXFP8 (native W4A8 mode: quantised every step)"} if args.w4a8 else {})),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"each step: the full route + combine and the fp64 grouped GEMM of both "
                                   f"projections on the first {n_slice} weight rows"},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
