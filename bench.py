#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 linear on B200.

Headline workload (one step): the four linears of one H3 ViT decoder block with 8
spatial tiles of 4096 tokens batched -- qkv [3072,1024], attn-out [1024,1024], FFN-in
[4096,1024], FFN-out [1024,4096], M = 32768 -- each with a 128-wide block Hadamard folded
into the weight, the dynamic activation scale (per-call amax), bias, bf16 output.  Per
linear the step runs the whole path: rotate + amax pass, rotate + quantize pass
(nvfp4_quantize) and the block-scaled GEMM (nvfp4_gemm_prepared, the weight scales
prepared offline with the packing), exactly the launches nvfp4_linear_prepared makes.
The K timed steps run back to back; a second pass with CUDA events between the launches
times the quantizer and the GEMM separately.  Inputs are seeded synthetic tensors already
in HBM; the activations of one step (448 MiB) exceed the 126 MB L2.

The other workloads of the pages are measured in the same run, one leg each:
  tiny          128 x 256 x 256, dynamic scale (launch-bound);
  static_scale  the headline step with a stored (calibrated) activation scale;
  qwen3_layer   the seven Qwen3-VL text-encoder projections at M = 512, dynamic scale;
  down_proj     SwiGLU input [4096, 25600] x [5120, 25600], g in {none, 16, 128}, with the
                relative error against the bf16 product;
  linear_m_sweep  nvfp4_linear at K = N = 5120, M in {16, 128, 1024, 8192, 65536};
  gemm_m_sweep  the GEMM alone over the same M (its HBM / tensor roofline);
  weight_pack   offline packing of one Qwen3-VL layer (487.6 M values);
  dequant, fused_chain, int8_linear  the rows-f paths;
  e2e           the headline step through nvfp4_linear_prepared with pinned host
                buffers: host-to-device copies, the linears and device-to-host copies on
                three streams, overlapped across the four linears and two buffers.
The CPU baseline is the oracle on a bounded row sample.

Prints one JSON line (rank 0).  --impl reference times the oracle instead; --leg NAME
runs one leg alone (for profiler captures).  Multi-GPU (torchrun): every rank runs its
own independent batch (weak scaling, no collective on the data path); timing is the max
over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nvfp4_block_scaled_17_b200 as nv  # noqa: E402
from nvfp4_block_scaled_17_b200 import workloads as W  # noqa: E402

METRIC = "nvfp4_linear TFLOPS (% of dense FP4 peak); quantizer GB/s (% of HBM)"

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one headline step's
# launches (4 GEMMs, 8 quantizer passes) from an ncu capture of `bench.py --kernels-only`
# with --cache-control none (L2 kept warm between launches, as in the timed loop).  Valid
# only for the kernel sources it was taken on (sha256 prefix); reported as null once a
# source has changed.
MEASURED_TRAFFIC = {
    "gemm": {"src": "nvfp4_block_scaled_17_b200/csrc/gemm.cu", "sha": "60b7b75abde4f94f",
             "bytes_per_step": 659.2e6},
    "quant": {"src": "nvfp4_block_scaled_17_b200/csrc/quantize.cu", "sha": "5c6efd3a218a6c59",
              "bytes_per_step": 824.3e6},
}

GROUP = 128
TOKENS = 8 * 4096
CPU_SAMPLE_ROWS = 16384
REF_SAMPLE_ROWS = 1024


def measured_traffic(key):
    t = MEASURED_TRAFFIC[key]
    try:
        sha = hashlib.sha256(open(os.path.join(ROOT, t["src"]), "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    return t["bytes_per_step"] if t["sha"] and sha == t["sha"] else None


def peaks():
    """Measured denominators.  The dense FP4 peak is not measured on this machine: it is
    taken as 4 x the measured bf16 GEMM (the nominal dense ratio 9 / 2.25), the burst
    figure for the short timed regions here, with the sustained one reported beside it."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        pk = {"hbm": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
              "bf16_sus": float(p["bf16_tflops_sustained"]), "src": "measured"}
    except Exception:
        pk = {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}
    pk["fp4"] = 4.0 * pk["bf16"]
    pk["fp4_sus"] = 4.0 * pk["bf16_sus"]
    return pk


def workload_config(act_scale: str):
    return {
        "workload": "vit_decoder_block_8tiles",
        "tokens": TOKENS,
        "linears": [f"{n}[{N}x{K}]" for n, N, K in W.VIT_SHAPES],
        "rotate_group": GROUP,
        "act_scale": act_scale,
        "bias": True,
        "l2": "inputs larger than L2 (448 MiB of activations per step, 126 MB L2)",
    }


def ev():
    return torch.cuda.Event(enable_timing=True)


def time_loop(fn, reps: int, warmup: int = 3) -> float:
    """Mean ms per call of `reps` back-to-back calls (events around the loop)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = ev(), ev()
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def time_each(fn, reps: int, flush: torch.Tensor | None = None, warmup: int = 3) -> float:
    """Mean ms of `reps` calls, each bracketed by events; with `flush`, a write of that
    buffer (larger than L2) precedes every call."""
    for _ in range(warmup):
        fn()
    pairs = [(ev(), ev()) for _ in range(reps)]
    for e0, e1 in pairs:
        if flush is not None:
            flush.fill_(1.0)
        e0.record()
        fn()
        e1.record()
    torch.cuda.synchronize()
    return sum(e0.elapsed_time(e1) for e0, e1 in pairs) / reps


def time_graph(fn, reps: int, flush: torch.Tensor | None = None) -> float | None:
    """Mean ms of one call inside a CUDA graph of `reps` calls (each after a write of
    `flush`, larger than L2, when given), minus the same graph without the calls: the
    device time without the host's per-call launch cost.  None if the call cannot be
    captured."""
    def capture(with_call):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            fn()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s):
                for _ in range(reps):
                    if flush is not None:
                        flush.fill_(1.0)
                    if with_call:
                        fn()
        torch.cuda.synchronize()
        return g

    try:
        g1, g0 = capture(True), (capture(False) if flush is not None else None)
    except Exception:
        torch.cuda.synchronize()
        return None

    def run(g):
        g.replay()
        torch.cuda.synchronize()
        a, b = ev(), ev()
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    t1 = min(run(g1) for _ in range(3))
    t0 = min(run(g0) for _ in range(3)) if g0 is not None else 0.0
    del g1, g0
    return (t1 - t0) / reps


def l2_flush_buffer(dev):
    return torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MiB


def linear_bytes(M, N, K, dynamic, l2):
    """Algorithmic HBM bytes of one linear: the quantizer reads x (twice with a dynamic
    scale once 2 * M * K > L2 / 2) and writes codes + scales; the GEMM reads them and
    the packed weight with its scales and writes bf16 y."""
    n = M * K
    reads = 2.0 if (dynamic and 2 * n > l2 // 2) else 1.0
    quant = n * (2.0 * reads + 0.5625)
    gemm = n * 0.5625 + N * K * 0.5625 + 2.0 * M * N
    return quant + gemm, quant, gemm


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        rows = [ln.split(",") for ln in open(self.file.name).read().strip().splitlines() if ln.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the headline step
# ---------------------------------------------------------------------------

class Layer:
    def __init__(self, lin: W.Linear, dev, group=GROUP):
        self.lin = lin
        self.group = group
        self.N, self.K = lin.N, lin.K
        self.M = lin.x.shape[0]
        self.x = lin.x
        self.bias = lin.bias
        self.wp, self.wsf, self.gsf_w = nv.pack_weight(lin.weight, group)
        # offline, with the packing: the weight scales in the order the GEMM copies them
        self.wsf_prep = nv.prepare_weight_scales(self.wsf, self.N, self.K)
        self.xp = torch.empty(self.M, self.K // 2, dtype=torch.uint8, device=dev)
        self.xsf = torch.empty(max(nv.nvfp4_scale_bytes(self.M, self.K), 1), dtype=torch.uint8,
                               device=dev)
        self.scalars = torch.empty(2, dtype=torch.float32, device=dev)
        self.ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
        self.y = torch.empty(self.M, self.N, dtype=torch.bfloat16, device=dev)
        self.lin_ws = torch.empty(nv.nvfp4_linear_workspace_bytes(self.M, self.K),
                                  dtype=torch.uint8, device=dev)
        self.gsf_static = None

    def flops(self):
        return 2.0 * self.M * self.N * self.K

    def quant_bytes(self, dynamic: bool, l2_bytes: int):
        n = self.M * self.K
        reads = 2.0 if (dynamic and 2 * n > l2_bytes // 2) else 1.0
        return n * (2.0 * reads + 0.5) + nv.nvfp4_scale_bytes(self.M, self.K)

    def quantize(self, dynamic: bool, stream=None):
        L = nv.lib()
        gsf_in = None if dynamic else self.gsf_static
        st = L.nvfp4_quantize(nv._ptr(self.x), self.M, self.K, self.group, nv._ptr(gsf_in),
                              nv._ptr(self.scalars[:1]), nv._ptr(self.xp), nv._ptr(self.xsf),
                              nv._ptr(self.gsf_w), nv._ptr(self.scalars[1:]), nv._ptr(self.ws),
                              self.ws.numel(), nv._stream(stream))
        if st:
            raise nv.NVFP4Error("nvfp4_quantize", st)

    def gemm(self, stream=None):
        st = nv.lib().nvfp4_gemm_prepared(nv._ptr(self.xp), nv._ptr(self.xsf), nv._ptr(self.wp),
                                          nv._ptr(self.wsf_prep), nv._ptr(self.scalars[1:]),
                                          nv._ptr(self.bias), nv._ptr(self.y), self.M, self.N,
                                          self.K, nv._stream(stream))
        if st:
            raise nv.NVFP4Error("nvfp4_gemm_prepared", st)

    def linear(self, dynamic: bool = True):
        """The public call: nvfp4_linear_prepared."""
        nv.nvfp4_linear(self.x, self.wp, self.wsf_prep, self.gsf_w, self.N, bias=self.bias,
                        gsf_x=None if dynamic else self.gsf_static, rotate_group=self.group,
                        workspace=self.lin_ws, out=self.y, prepared=True)


def run_step(layers, dynamic: bool, events=None):
    """One pass of the path over the linears -- the same two entry points and launches
    per linear that nvfp4_linear_prepared makes (quantize writing alpha, then the GEMM);
    events[i] = (e0, e1, e2) per linear bracket the quantizer and the GEMM."""
    for i, ly in enumerate(layers):
        if events is not None:
            events[i][0].record()
        ly.quantize(dynamic)
        if events is not None:
            events[i][1].record()
        ly.gemm()
        if events is not None:
            events[i][2].record()


def timed_steps(layers, dynamic, steps, warmup, dist_on):
    """The K timed steps with nothing between the launches (start/stop events only, so
    consecutive kernels can overlap their launch and set-up), then the same K steps once
    more with an event around every launch for the per-kernel durations."""
    for _ in range(warmup):
        run_step(layers, dynamic)
    start, stop = ev(), ev()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record()
    for _ in range(steps):
        run_step(layers, dynamic)
    stop.record()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(stop)
    evs = [[[ev() for _ in range(3)] for _ in layers] for _ in range(steps)]
    for k in range(steps):
        run_step(layers, dynamic, evs[k])
    torch.cuda.synchronize()
    q_ms = [sum(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(steps)) / steps
            for i in range(len(layers))]
    g_ms = [sum(evs[k][i][1].elapsed_time(evs[k][i][2]) for k in range(steps)) / steps
            for i in range(len(layers))]
    return total_ms, q_ms, g_ms


def quantizer_launches(M, K, group, dynamic, sms=148):
    """Kernel launches one nvfp4_quantize call makes: one for a static scale, for a dynamic
    call of at most 12 items of 32 units (the one-CTA single pass), or for an unrotated
    dynamic call on rows of whole 128-value units (amax and encode phases in one kernel);
    two (amax pass, encode pass) for other dynamic calls."""
    if not dynamic:
        return 1
    if K % 128 == 0:
        items = -(-(M * (K // 128)) // 32)
        if items <= 12 or group == 0:
            return 1
    return 2


def max_over_ranks(v: float, dist_on: bool) -> float:
    """The slowest rank's figure (a device tensor under NCCL, a host one under gloo)."""
    if not dist_on:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own batch of
    the same size, so the job does world x the per-rank work in the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def rank_seed(rank: int) -> int:
    """Each rank draws its own independent batch."""
    return 1001 + rank


# ---------------------------------------------------------------------------
# end to end through the public call, copies overlapped
# ---------------------------------------------------------------------------

def e2e_steps(layers, steps, warmup, dist_on):
    """Per step: host-to-device copy of every linear's x from pinned memory, the linear
    (nvfp4_linear_prepared), device-to-host copy of every y into pinned memory.  Copies
    in each direction run on their own stream and the linears on a third, ordered by
    events; the device buffers alternate between two sets, so the upload of step k+1 and
    the download of step k - 1 overlap the linears of step k.  Timed on the device from
    the first upload to the last download."""
    comp = torch.cuda.current_stream()
    s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
    host_x = [ly.x.cpu().pin_memory() for ly in layers]
    host_y = [torch.empty(ly.y.shape, dtype=torch.bfloat16).pin_memory() for ly in layers]
    dev_x = [[torch.empty_like(ly.x) for ly in layers] for _ in range(2)]
    dev_y = [[torch.empty_like(ly.y) for ly in layers] for _ in range(2)]
    n = len(layers)
    x_ready = [[ev() for _ in range(n)] for _ in range(2)]
    x_free = [[ev() for _ in range(n)] for _ in range(2)]
    y_ready = [[ev() for _ in range(n)] for _ in range(2)]
    y_free = [[ev() for _ in range(n)] for _ in range(2)]

    def step(k):
        b = k % 2
        for i in range(n):
            if k >= 2:
                s_up.wait_event(x_free[b][i])
            with torch.cuda.stream(s_up):
                dev_x[b][i].copy_(host_x[i], non_blocking=True)
            x_ready[b][i].record(s_up)
        for i, ly in enumerate(layers):
            comp.wait_event(x_ready[b][i])
            if k >= 2:
                comp.wait_event(y_free[b][i])
            nv.nvfp4_linear(dev_x[b][i], ly.wp, ly.wsf_prep, ly.gsf_w, ly.N, bias=ly.bias,
                            rotate_group=ly.group, workspace=ly.lin_ws, out=dev_y[b][i],
                            prepared=True, stream=comp)
            x_free[b][i].record(comp)
            y_ready[b][i].record(comp)
        for i in range(n):
            s_down.wait_event(y_ready[b][i])
            with torch.cuda.stream(s_down):
                host_y[i].copy_(dev_y[b][i], non_blocking=True)
            y_free[b][i].record(s_down)

    k = 0
    for _ in range(warmup):
        step(k)
        k += 1
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    start, stop = ev(), ev()
    start.record(s_up)
    comp.wait_event(start)
    s_down.wait_event(start)
    for _ in range(steps):
        step(k)
        k += 1
    comp.wait_stream(s_up)
    comp.wait_stream(s_down)
    stop.record(comp)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    ms = max_over_ranks(start.elapsed_time(stop) / steps, dist_on)
    h2d = sum(x.numel() * 2 for x in host_x)
    d2h = sum(y.numel() * 2 for y in host_y)
    # the copies alone, for the bound: each direction timed by itself
    up_ms = time_loop(lambda: [dev_x[0][i].copy_(host_x[i], non_blocking=True) for i in range(n)], 3, 1)
    down_ms = time_loop(lambda: [host_y[i].copy_(dev_y[0][i], non_blocking=True) for i in range(n)], 3, 1)
    del dev_x, dev_y
    return ms, h2d, d2h, up_ms, down_ms


# ---------------------------------------------------------------------------
# the other workloads
# ---------------------------------------------------------------------------

def leg_tiny(dev, pk, l2):
    """The tiny linear (x [128, 256] with 1 % outliers x20, W [256, 256], bias, dynamic
    scale, no rotation) through nvfp4_linear: launch-bound, timed as back-to-back calls."""
    lin = W.tiny(dev)
    ly = Layer(lin, dev, group=0)
    ms_eager = time_loop(lambda: ly.linear(True), 200, 10)
    ms_graph = time_graph(lambda: ly.linear(True), 50)
    ms = ms_graph if ms_graph is not None else ms_eager
    f = ly.flops()
    return {"workload": "tiny W4A4 linear 128 x 256 x 256, dynamic scale, bias",
            "us": ms * 1e3, "TFLOP/s": f / (ms * 1e-3) / 1e12, "eager_us": ms_eager * 1e3,
            "timing": "CUDA graph of 50 calls back to back" if ms_graph is not None else "eager",
            "launches": quantizer_launches(128, 256, 0, True) + 1,
            "note": "launch-bound: 16.8 MFLOP per call"}


def leg_qwen3_layer(dev, pk, l2):
    """The seven Qwen3-VL-32B projections of one text-encoder layer at M = 512 (dynamic
    scale, no bias, no rotation) through nvfp4_linear_prepared, back to back; the weights
    (274 MB packed) exceed L2.  Per projection a second pass times the quantizer and the
    GEMM with events between them."""
    layers = [Layer(l, dev, group=0) for l in W.qwen3_layer(dev)]
    reps = 10

    def layer_step():
        for ly in layers:
            ly.linear(True)

    ms = time_loop(layer_step, reps, 3)
    evs = [[[ev() for _ in range(3)] for _ in layers] for _ in range(reps)]
    for k in range(reps):
        run_step(layers, True, evs[k])
    torch.cuda.synchronize()
    per = []
    for i, ly in enumerate(layers):
        q = sum(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(reps)) / reps
        g = sum(evs[k][i][1].elapsed_time(evs[k][i][2]) for k in range(reps)) / reps
        tf = ly.flops() / (g * 1e-3) / 1e12
        tot, _, gb = linear_bytes(ly.M, ly.N, ly.K, True, l2)
        per.append({"proj": ly.lin.name, "N": ly.N, "K": ly.K, "quantizer_us": q * 1e3,
                    "gemm_us": g * 1e3, "gemm_TFLOP/s": tf, "gemm_frac_of_fp4_peak": tf / pk["fp4"],
                    "gemm_GBps": gb / (g * 1e-3) / 1e9})
    flops = sum(ly.flops() for ly in layers)
    tf = flops / (ms * 1e-3) / 1e12
    del layers
    return {"workload": "Qwen3-VL-32B text-encoder layer, 7 projections, M = 512, dynamic scale",
            "ms": ms, "TFLOP/s": tf, "frac_of_fp4_peak": tf / pk["fp4"],
            "launches_per_layer": 7 * (quantizer_launches(512, 5120, 0, True) + 1),
            "per_projection": per}


def leg_down_proj(dev, pk, l2):
    """down_proj with the SwiGLU / Student-t(3) input, [4096, 25600] x [5120, 25600], no
    bias, dynamic scale, for g in {none, 16, 128}: nvfp4_linear_prepared time, the
    quantizer / GEMM split, and the relative error of the output against the product of
    the bf16 operands (fp64 on 256 sampled rows)."""
    lin = W.down_proj_swiglu(dev)
    rows = torch.randperm(lin.x.shape[0], generator=W._gen(7, "cpu"))[:256].to(dev)
    ref = lin.x[rows].double() @ lin.weight.double().t()
    out = []
    for g in (0, 16, 128):
        ly = Layer(lin, dev, group=g)
        ms = time_loop(lambda: ly.linear(True), 10, 3)
        evs = [[[ev() for _ in range(3)]] for _ in range(5)]
        for k in range(5):
            run_step([ly], True, evs[k])
        torch.cuda.synchronize()
        q = sum(e[0][0].elapsed_time(e[0][1]) for e in evs) / 5
        gm = sum(e[0][1].elapsed_time(e[0][2]) for e in evs) / 5
        ly.linear(True)
        err = float((ly.y[rows].double() - ref).norm() / ref.norm())
        tf = ly.flops() / (ms * 1e-3) / 1e12
        gtf = ly.flops() / (gm * 1e-3) / 1e12
        out.append({"rotate_group": g, "ms": ms, "TFLOP/s": tf, "quantizer_ms": q,
                    "gemm_ms": gm, "gemm_TFLOP/s": gtf, "gemm_frac_of_fp4_peak": gtf / pk["fp4"],
                    "rel_err_vs_bf16_product": err})
        del ly
    del lin, ref
    return {"workload": "down_proj 4096 x 5120 x 25600, SwiGLU input (0.5 Student-t(3) factors), "
                        "dynamic scale", "per_group": out}


def leg_linear_m_sweep(dev, pk, l2):
    """nvfp4_linear_prepared at N = K = 5120 over M in {16, 128, 1024, 8192, 65536}: an
    N(0, 0.02) weight packed offline, x ~ N(0, 1), dynamic scale, no bias; each call
    timed alone after a write larger than L2.  Against the FP4 peak and against the HBM
    roofline over the linear's algorithmic bytes (quantizer + GEMM)."""
    flush = l2_flush_buffer(dev)
    pts = []
    for M in W.M_SWEEP:
        lin = W.m_sweep(M, dev)
        ly = Layer(lin, dev, group=0)
        ms_eager = time_each(lambda: ly.linear(True), 10, flush)
        ms_graph = time_graph(lambda: ly.linear(True), 10, flush)
        ms = ms_graph if ms_graph is not None else ms_eager
        tot, qb, gb = linear_bytes(M, 5120, 5120, True, l2)
        tf = ly.flops() / (ms * 1e-3) / 1e12
        gbps = tot / (ms * 1e-3) / 1e9
        pts.append({"M": M, "us": ms * 1e3, "TFLOP/s": tf, "frac_of_fp4_peak": tf / pk["fp4"],
                    "GBps": gbps, "frac_of_hbm": gbps / pk["hbm"], "eager_us": ms_eager * 1e3,
                    "timing": "graph" if ms_graph is not None else "eager",
                    "launches": quantizer_launches(M, 5120, 0, True) + 1})
        del ly, lin
    del flush
    return {"workload": "nvfp4_linear_prepared, N = K = 5120, dynamic scale, no bias, L2 "
                        "flushed before each call; us from a CUDA graph of flush + call pairs "
                        "minus the flushes alone (eager_us: events around each eager call)",
            "points": pts}


def leg_gemm_m_sweep(dev, pk, l2):
    """nvfp4_gemm_prepared at N = K = 5120 over M in {16, 128, 1024, 8192, 65536} (no
    bias), each launch timed alone after a write of 256 MiB (more than L2).  Random
    packed operands with finite E4M3 block scales (0.5 .. 0.94).  Small M is bound by the
    weight stream, so every point is also given against the HBM roofline over
    N*K*(0.5 + 1/16) + M*K*(0.5 + 1/16) + 2*M*N bytes."""
    N = K = 5120
    g = torch.Generator(device=dev).manual_seed(1005)

    def operand(rows):
        packed = torch.randint(0, 256, (rows, K // 2), generator=g, device=dev,
                               dtype=torch.int32).to(torch.uint8)
        sf = (0x30 + torch.randint(0, 16, (nv.nvfp4_scale_bytes(rows, K),), generator=g,
                                   device=dev, dtype=torch.int32)).to(torch.uint8)
        return packed, sf

    wp, wsf = operand(N)
    wsf = nv.prepare_weight_scales(wsf, N, K)
    alpha = torch.tensor([1e-3], device=dev)
    flush = l2_flush_buffer(dev)
    points = []
    for M in W.M_SWEEP:
        xp, xsf = operand(M)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        call = lambda: nv.nvfp4_gemm_prepared(xp, xsf, wp, wsf, alpha, None, M, N, K, out=y)
        ms_eager = time_each(call, 10, flush)
        ms_graph = time_graph(call, 10, flush)
        ms = ms_graph if ms_graph is not None else ms_eager
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        gb = (N * K * 0.5625 + M * K * 0.5625 + 2.0 * M * N) / (ms * 1e-3) / 1e9
        points.append({"M": M, "us": ms * 1e3, "TFLOP/s": tf,
                       "frac_of_fp4_peak": tf / pk["fp4"], "GBps": gb,
                       "frac_of_hbm": gb / pk["hbm"], "eager_us": ms_eager * 1e3,
                       "timing": "graph" if ms_graph is not None else "eager"})
        del xp, xsf, y
    del flush
    return {"workload": "nvfp4_gemm_prepared, N = K = 5120, no bias, L2 flushed before each "
                        "launch; us from a CUDA graph of flush + call pairs minus the flushes "
                        "alone (eager_us: events around each eager call)", "points": points}


def leg_gemm_square(dev, pk, l2):
    """The GEMM alone at 8192 x 8192 x 8192 (no bias), with 128x4 and with prepared weight
    scales: each launch timed by events after a write of 256 MiB (more than L2).  Random
    packed operands with finite E4M3 block scales (0.5 .. 0.94); 1.1 TFLOP per launch."""
    M = N = K = 8192
    g = torch.Generator(device=dev).manual_seed(1007)

    def operand(rows):
        packed = torch.randint(0, 256, (rows, K // 2), generator=g, device=dev,
                               dtype=torch.int32).to(torch.uint8)
        sf = (0x30 + torch.randint(0, 16, (nv.nvfp4_scale_bytes(rows, K),), generator=g,
                                   device=dev, dtype=torch.int32)).to(torch.uint8)
        return packed, sf

    xp, xsf = operand(M)
    wp, wsf = operand(N)
    wsf_p = nv.prepare_weight_scales(wsf, N, K)
    alpha = torch.tensor([1e-3], device=dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    flush = l2_flush_buffer(dev)
    out = {"workload": "nvfp4_gemm / nvfp4_gemm_prepared at 8192^3, no bias, L2 flushed "
                       "before each launch, 20 launches after 3 warm-up"}
    for name, call in (
            ("128x4", lambda: nv.nvfp4_gemm(xp, xsf, wp, wsf, alpha, None, M, N, K, out=y)),
            ("prepared", lambda: nv.nvfp4_gemm_prepared(xp, xsf, wp, wsf_p, alpha, None, M, N,
                                                        K, out=y))):
        ms = time_each(call, 20, flush)
        tf = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[name] = {"us": ms * 1e3, "TFLOP/s": tf, "frac_of_fp4_peak": tf / pk["fp4"]}
    del flush
    return out


def leg_weight_pack(dev, pk, l2):
    """Offline weight packing at the text-encoder scale: the seven Qwen3-VL projection
    shapes of one layer (487.6 M values, N(0, 0.02), generated untimed), each quantized with
    its own dynamic global scale into preallocated outputs, then once more under that
    scale as a static one (the encode pass alone).  GB/s over 4.5625 B/value where
    2 * numel > L2 / 2 (x read twice) and 2.5625 B/value otherwise, plus the scale bytes.
    The 50-layer pack (24.4 B values) is given as 50 x this layer's time."""
    g = W._gen(1005, dev)
    items = []
    for name, N, K in W.QWEN3_SHAPES:
        w = W.qwen3_weight((N, K), dev, g)
        packed = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
        sf = torch.empty(nv.nvfp4_scale_bytes(N, K), dtype=torch.uint8, device=dev)
        gsf = torch.empty(1, dtype=torch.float32, device=dev)
        items.append((name, w, packed, sf, gsf))
    ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(), dtype=torch.uint8, device=dev)

    # Each rep enqueues all seven calls with an event pair around each, largest tensors
    # first; rep 0 is discarded.  The host then runs ahead of the GPU (the 131 M-value
    # projections take about 100 us each), so every event pair times the GPU alone.
    order = sorted(items, key=lambda it: -it[1].numel())
    reps = 4

    def run(static: bool, g_static=None):
        evs = [[(ev(), ev()) for _ in order] for _ in range(reps)]
        for r in range(reps):
            for j, (name, w, packed, sf, gsf) in enumerate(order):
                g_in = g_static[j] if static else None
                evs[r][j][0].record()
                nv.nvfp4_quantize(w, 0, g_in, out=(packed, sf, gsf), workspace=ws)
                evs[r][j][1].record()
        torch.cuda.synchronize()
        return [sum(evs[r][j][0].elapsed_time(evs[r][j][1]) for r in range(1, reps)) / (reps - 1)
                for j in range(len(order))]

    ms_dyn = run(False)
    g_static = [it[4].clone() for it in order]
    ms_st = run(True, g_static)
    per, n_all, b_dyn, b_st, t_dyn, t_st = [], 0, 0.0, 0.0, 0.0, 0.0
    for (name, w, packed, sf, gsf), ms_d, ms_s in zip(order, ms_dyn, ms_st):
        n = w.numel()
        bpv = 4.5625 if 2 * n > l2 / 2 else 2.5625
        by_d = n * bpv + sf.numel()
        by_s = n * 2.5625 + sf.numel()
        per.append({"tensor": name, "values": n, "dynamic_us": ms_d * 1e3,
                    "dynamic_GBps": by_d / (ms_d * 1e-3) / 1e9, "bytes_per_value": bpv,
                    "static_us": ms_s * 1e3, "static_GBps": by_s / (ms_s * 1e-3) / 1e9})
        n_all += n
        b_dyn += by_d
        b_st += by_s
        t_dyn += ms_d
        t_st += ms_s
    del items, ws
    gb_d = b_dyn / (t_dyn * 1e-3) / 1e9
    gb_s = b_st / (t_st * 1e-3) / 1e9
    return {"workload": "Qwen3-VL-32B text-encoder layer, 7 projections, dynamic scale each",
            "values": n_all, "ms": t_dyn, "GBps": gb_d, "frac_of_measured_hbm": gb_d / pk["hbm"],
            "frac_of_8TBps": gb_d / 8000.0,
            "static_ms": t_st, "static_GBps": gb_s,
            "static_frac_of_measured_hbm": gb_s / pk["hbm"],
            "pack_50_layers_s": 50 * t_dyn * 1e-3, "per_tensor": per}


def leg_fused_chain(dev, pk, l2):
    """The FFN pair of the block (FFN in [4096 x 1024] then FFN out [1024 x 4096], M = 32768)
    on the static-scale path the pages fuse (no rotation, precomputed global scales):
    unfused = quantize x, GEMM 1 -> bf16 y1, quantize y1, GEMM 2; fused = quantize x,
    GEMM 1 with the NVFP4 encoding of y1 as its output, GEMM 2.  Scales are calibrated
    from one dynamic call on this input (untimed)."""
    src = W.vit_block(dev)
    l1, l2_ = src[2], src[3]
    M, N1, K1, N2 = l1.x.shape[0], l1.N, l1.K, l2_.N
    w1p, w1sf, g1w = nv.pack_weight(l1.weight, 0)
    w2p, w2sf, g2w = nv.pack_weight(l2_.weight, 0)
    x = l1.x
    xp, xsf, gx = nv.nvfp4_quantize(x, 0, None)
    a1 = 1.0 / (gx * g1w)
    y1 = nv.nvfp4_gemm(xp, xsf, w1p, w1sf, a1, l1.bias, M, N1, K1)
    _, _, gy = nv.nvfp4_quantize(y1, 0, None)
    a2 = 1.0 / (gy * g2w)
    y1p = torch.empty(M, N1 // 2, dtype=torch.uint8, device=dev)
    y1sf = torch.empty(nv.nvfp4_scale_bytes(M, N1), dtype=torch.uint8, device=dev)
    g_tmp = torch.empty(1, dtype=torch.float32, device=dev)
    y2 = torch.empty(M, N2, dtype=torch.bfloat16, device=dev)

    def unfused():
        nv.nvfp4_quantize(x, 0, gx, out=(xp, xsf, g_tmp))
        nv.nvfp4_gemm(xp, xsf, w1p, w1sf, a1, l1.bias, M, N1, K1, out=y1)
        nv.nvfp4_quantize(y1, 0, gy, out=(y1p, y1sf, g_tmp))
        nv.nvfp4_gemm(y1p, y1sf, w2p, w2sf, a2, l2_.bias, M, N2, N1, out=y2)

    def fused():
        nv.nvfp4_quantize(x, 0, gx, out=(xp, xsf, g_tmp))
        nv.nvfp4_gemm_quantize_out(xp, xsf, w1p, w1sf, a1, M, N1, K1, gy, bias=l1.bias,
                                   out=(y1p, y1sf))
        nv.nvfp4_gemm(y1p, y1sf, w2p, w2sf, a2, l2_.bias, M, N2, N1, out=y2)

    t_un, t_fu = time_loop(unfused, 10), time_loop(fused, 10)
    t_g = time_loop(lambda: nv.nvfp4_gemm_quantize_out(xp, xsf, w1p, w1sf, a1, M, N1, K1, gy,
                                                       bias=l1.bias, out=(y1p, y1sf)), 10)
    flops = 2.0 * M * N1 * K1 + 2.0 * M * N2 * N1
    return {"workload": "ViT FFN pair, M=32768, static scales, no rotation",
            "unfused_ms": t_un, "fused_ms": t_fu, "speedup": t_un / t_fu,
            "unfused_TFLOPs": flops / (t_un * 1e-3) / 1e12,
            "fused_TFLOPs": flops / (t_fu * 1e-3) / 1e12,
            "fused_gemm_ms": t_g,
            "fused_gemm_TFLOPs": 2.0 * M * N1 * K1 / (t_g * 1e-3) / 1e12}


def leg_int8(dev, pk, l2):
    """The same four ViT-block linears (M = 32768) on the int8 per-row W8A8 path: per
    linear, the per-row activation quantizer then the int8 GEMM (weights quantized
    offline, untimed).  TOPS against the int8 dense peak (2 x the measured bf16 burst
    figure, nominal ratio 4.5 / 2.25); the quantizer's GB/s over 2 B read + 1 B + 4 B / row
    written."""
    layers = []
    for l in W.vit_block(dev):
        wq, sw = nv.int8_quantize_rows(l.weight)
        M, K = l.x.shape
        layers.append(dict(x=l.x, wq=wq, sw=sw, bias=l.bias, M=M, K=K, N=l.N,
                           xq=torch.empty(M, K, dtype=torch.int8, device=dev),
                           sx=torch.empty(M, dtype=torch.float32, device=dev),
                           y=torch.empty(M, l.N, dtype=torch.bfloat16, device=dev)))

    def step(evs=None):
        for i, L_ in enumerate(layers):
            if evs is not None:
                evs[i][0].record()
            nv.int8_quantize_rows(L_["x"], out=(L_["xq"], L_["sx"]))
            if evs is not None:
                evs[i][1].record()
            nv.int8_gemm(L_["xq"], L_["sx"], L_["wq"], L_["sw"], L_["bias"], out=L_["y"])
            if evs is not None:
                evs[i][2].record()

    ms = time_loop(step, 10)
    reps = 10
    evs = [[[ev() for _ in range(3)] for _ in layers] for _ in range(reps)]
    for k in range(reps):
        step(evs[k])
    torch.cuda.synchronize()
    q_ms = sum(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(reps) for i in range(4)) / reps
    g_ms = sum(evs[k][i][1].elapsed_time(evs[k][i][2]) for k in range(reps) for i in range(4)) / reps
    ops = sum(2.0 * L_["M"] * L_["N"] * L_["K"] for L_ in layers)
    qbytes = sum(L_["M"] * L_["K"] * 3.0 + L_["M"] * 4.0 for L_ in layers)
    i8_peak = 2.0 * pk["bf16"]
    g_tops = ops / (g_ms * 1e-3) / 1e12
    return {"workload": "ViT block linears, M=32768, int8 per-row W8A8",
            "ms_per_step": ms, "TOPS": ops / (ms * 1e-3) / 1e12,
            "gemm_ms": g_ms, "gemm_TOPS": g_tops, "gemm_frac_of_int8_peak": g_tops / i8_peak,
            "int8_peak_TOPS": i8_peak, "quantizer_ms": q_ms,
            "quantizer_GBps": qbytes / (q_ms * 1e-3) / 1e9,
            "quantizer_frac_of_hbm": qbytes / (q_ms * 1e-3) / 1e9 / pk["hbm"]}


def leg_dequant(dev, pk, l2):
    """NVFP4 -> bf16 expansion of one 5120 x 25600 projection (131 M values; 74 MB in,
    262 MB out, above L2), GB/s over the algorithmic 0.5 + 1/16 + 2 = 2.5625 B/value.  The
    packed weight is an N(0, 0.02) weight quantized by nvfp4_quantize (untimed)."""
    rows, K = 5120, 25600
    w = W.qwen3_weight((rows, K), dev, W._gen(1005, dev))
    packed, sf, gsf = nv.nvfp4_quantize(w, 0, None)
    del w
    y = torch.empty(rows, K, dtype=torch.bfloat16, device=dev)
    ms = time_loop(lambda: nv.nvfp4_dequantize(packed, sf, gsf, K, out=y), 10)
    n = rows * K
    gbps = n * 2.5625 / (ms * 1e-3) / 1e9
    return {"values": n, "ms": ms, "GBps": gbps, "bytes_per_value": 2.5625,
            "frac_of_measured_hbm": gbps / pk["hbm"]}


LEGS = {
    "tiny": leg_tiny,
    "qwen3_layer": leg_qwen3_layer,
    "down_proj": leg_down_proj,
    "linear_m_sweep": leg_linear_m_sweep,
    "gemm_m_sweep": leg_gemm_m_sweep,
    "gemm_square": leg_gemm_square,
    "weight_pack": leg_weight_pack,
    "dequant": leg_dequant,
    "fused_chain": leg_fused_chain,
    "int8_linear": leg_int8,
}


# ---------------------------------------------------------------------------
# CPU oracle
# ---------------------------------------------------------------------------

def oracle_pack(layers_src):
    """The oracle's own weight packing (rotate g=128, dynamic quantize); untimed."""
    import oracle as O
    O.build()
    return [O.quantize(O.hadamard_rotate(W.to_u16(l.weight), GROUP)) for l in layers_src]


def host_cores() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    if n:
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(layers_src, rows: int, packed=None):
    """The oracle as it stands on the host cores: rotate, dynamic quantize and the fp64
    GEMM for `rows` rows of each linear (weights packed by the oracle, untimed)."""
    import oracle as O
    if packed is None:
        packed = oracle_pack(layers_src)
    xs = [W.to_u16(l.x[:rows]) for l in layers_src]
    bs = [W.to_u16(l.bias) for l in layers_src]
    t0 = time.perf_counter()
    flops = 0.0
    for l, (wp, wsf, gw), x, b in zip(layers_src, packed, xs, bs):
        O.linear(x, wp, wsf, gw, l.N, b, rotate_group=GROUP)
        flops += 2.0 * rows * l.N * l.K
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": host_cores(),
            "kind": "oracle",
            "sample": f"{rows} rows of each of the 4 linears (rotate g=128, dynamic quantize, "
                      f"fp64 GEMM over all N), {dt:.1f} s"}, dt


# ---------------------------------------------------------------------------
# runs
# ---------------------------------------------------------------------------

def run_ours(args, dist_on, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 1024 * 1024))
    sms = props.multi_processor_count
    pk = peaks()
    src = W.vit_block(dev, seed=rank_seed(rank), tokens=TOKENS)
    layers = [Layer(l, dev) for l in src]
    # static scale: the scale a calibration pass over this very input would store, i.e.
    # the dynamic scale of one untimed call
    for ly in layers:
        _, _, g = nv.nvfp4_quantize(ly.x, GROUP, None)
        ly.gsf_static = g
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    if not args.kernels_only:
        clocks.start()
    total_ms, q_ms, g_ms = timed_steps(layers, True, args.steps, args.warmup, dist_on)
    clk = None if args.kernels_only else clocks.stop()
    legs = {}
    if not args.kernels_only:
        s_total, s_q, s_g = timed_steps(layers, False, args.steps, args.warmup, dist_on)
        # the same K steps as the kernel timing: the pipeline's fill and drain (the first
        # upload, the last download) are spread over all of them
        e2e_ms, h2d, d2h, up_ms, down_ms = e2e_steps(layers, args.steps, max(3, args.warmup),
                                                     dist_on)
        if world == 1:      # the other workloads: single-GPU runs only
            for name, fn in LEGS.items():
                legs[name] = fn(dev, pk, l2)
                torch.cuda.empty_cache()
    assert nv.last_device_status() == nv.OK

    ms = max_over_ranks(total_ms / args.steps, dist_on)
    flops = sum(ly.flops() for ly in layers)
    value = aggregate_tflops(flops, ms, world)

    g_time = sum(g_ms)
    gemm_tflops = flops / (g_time * 1e-3) / 1e12
    q_bytes = sum(ly.quant_bytes(True, l2) for ly in layers)
    q_time = sum(q_ms)
    q_gbps = q_bytes / (q_time * 1e-3) / 1e9
    dominant_is_gemm = g_time >= q_time
    g_bytes = sum(ly.M * ly.K * 0.5625 + ly.N * ly.K * 0.5625 + ly.M * ly.N * 2 for ly in layers)
    g_traffic, q_traffic = measured_traffic("gemm"), measured_traffic("quant")
    gemm_roof = {"bound": "tensor", "achieved": gemm_tflops, "peak": pk["fp4"], "unit": "TFLOP/s",
                 "frac": gemm_tflops / pk["fp4"], "traffic": g_traffic,
                 "traffic_unit": "DRAM bytes per step (4 launches)",
                 "algorithmic_bytes": g_bytes,
                 "traffic_over_algorithmic": g_traffic / g_bytes if g_traffic else None,
                 "algorithmic_flop": flops, "kernel": "gemm_kernel (prepared weight scales)",
                 "per_linear_ms": g_ms,
                 "peak_note": f"{pk['src']}: 4 x bf16 burst ({pk['bf16']} TFLOP/s), nominal dense "
                              "fp4/bf16 ratio 9/2.25; the timed region is a short burst",
                 "frac_of_sustained_peak": gemm_tflops / pk["fp4_sus"],
                 "frac_of_nominal_9PF": gemm_tflops / 9000.0}
    quant_roof = {"bound": "hbm", "achieved": q_gbps, "peak": pk["hbm"], "unit": "GB/s",
                  "frac": q_gbps / pk["hbm"], "traffic": q_traffic,
                  "traffic_unit": "DRAM bytes per step (8 launches)", "algorithmic_bytes": q_bytes,
                  "traffic_over_algorithmic": q_traffic / q_bytes if q_traffic else None,
                  "kernel": "row_kernel (amax pass + encode pass, g = 128)", "per_linear_ms": q_ms,
                  "bytes_note": "4.5625 B/value (two reads of x, dynamic scale, x > L2/2) + scales",
                  "peak_note": f"{pk['src']} copy bandwidth",
                  "frac_of_8TBps": q_gbps / 8000.0}
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3/16, fp32 accumulate)",
        "data": "synthetic (seeded; N(0,1) activations with 0.5% outliers x30, N(0,0.02) weights)",
        "config": workload_config("dynamic"),
        "roofline": gemm_roof if dominant_is_gemm else quant_roof,
        "roofline_gemm": gemm_roof, "roofline_quantizer": quant_roof,
        "gpu_launches": sum(quantizer_launches(ly.M, ly.K, GROUP, True, sms) + 1
                            for ly in layers) * args.steps,
        "clocks": clk,
    }
    if not args.kernels_only:
        n_vals = sum(ly.M * ly.K for ly in layers)
        enc_ms, amax_ms = sum(s_q), sum(q_ms) - sum(s_q)
        quant_roof["passes"] = {
            "encode_GBps": n_vals * 2.5625 / (enc_ms * 1e-3) / 1e9,
            "amax_GBps": n_vals * 2.0 / (amax_ms * 1e-3) / 1e9 if amax_ms > 0 else None,
            "note": "encode = the static-scale quantizer; amax = dynamic minus static"}
        s_ms = max_over_ranks(s_total / args.steps, dist_on)
        out["static_scale"] = {"ms_per_step": s_ms, "TFLOP/s": aggregate_tflops(flops, s_ms, world),
                               "quantizer_ms": s_q, "gemm_ms": s_g,
                               "dynamic_over_static_quantizer": sum(q_ms) / sum(s_q)}
        pcie_bound = max(up_ms, down_ms)
        out["e2e"] = {"value": aggregate_tflops(flops, e2e_ms, world), "unit": "TFLOP/s",
                      "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "api": "nvfp4_linear_prepared",
                      "copy_only_ms": {"h2d": up_ms, "d2h": down_ms},
                      "frac_of_copy_bound": pcie_bound / e2e_ms}
        out.update(legs)
    if rank == 0 and world == 1 and not (args.no_cpu_baseline or args.kernels_only):
        cb, _ = cpu_baseline(src, CPU_SAMPLE_ROWS)
        out["cpu_baseline"] = cb
    return out


def run_leg(name, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 1024 * 1024))
    res = LEGS[name](dev, peaks(), l2)
    assert nv.last_device_status() == nv.OK
    return {"leg": name, **res}


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is a bounded sample of the same
    workload (REF_SAMPLE_ROWS rows of each linear, about a second on the host cores);
    rank 0 only, the other ranks exit without work."""
    if rank != 0:
        return None
    src = W.vit_block("cpu", seed=1001, tokens=REF_SAMPLE_ROWS)
    packed = oracle_pack(src)
    for _ in range(args.warmup):
        cpu_baseline(src, 8, packed)
    vals, dts = [], []
    for _ in range(args.steps):
        cb, dt = cpu_baseline(src, REF_SAMPLE_ROWS, packed)
        vals.append(cb["value"])
        dts.append(dt)
    v = sum(2.0 * REF_SAMPLE_ROWS * l.N * l.K for l in src) * len(dts) / sum(dts) / 1e12
    cb["value"] = v
    cb["sample"] = (f"{REF_SAMPLE_ROWS} rows of each of the 4 linears per step (rotate g=128, "
                    f"dynamic quantize, fp64 GEMM over all N), {args.steps} steps")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(dts),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": workload_config("dynamic"),
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernels-only", action="store_true",
                    help="time only the dynamic-scale headline step (for profiler runs)")
    ap.add_argument("--leg", choices=sorted(LEGS), default=None,
                    help="run one leg alone and print its JSON (for profiler runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if args.leg:
        if rank == 0:
            print(json.dumps(run_leg(args.leg, local_rank)), flush=True)
        return
    if dist_on:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    out = run_ours(args, dist_on, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
