#!/usr/bin/env python
"""Benchmark of the INT8 quantized-training Linear layer on B200.

One step = one pass of the whole hot path over one batch: the 5376 -> 7168
layer of OneTrainer PR #1681 "Int8 conv rot" at 12000 tokens with Hadamard
block 128, bf16 X and dY:
    qlinear_fwd       per-row rotate + quantize X (saved int8), int8 GEMM, scale + bias -> bf16 y
    qlinear_bwd       from one shared preparation of dY (column statistics, then one pass
                      writing the row-quantized dY*s_w and the column-quantized dY*s_x):
                      int8 GEMM dY_q W_q, scale, fused rotation -> bf16 dX, and
                      int8 GEMM dY_q^T X_q, scale -> fp32 dW; db
    qweight_update_sr AdamW on the int8 weight + Philox stochastic requantization
Metric: int8 tensor operations of the three GEMMs (3 x 2*M*N*K) per second,
in TOPS, whole job (all ranks).  Inputs stay resident in HBM; the step's
working set (about 1 GB) is far larger than the 126 MB L2.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With N > 1 it runs under torchrun, one independent replica per GPU (the
layer's path has no exchange step), and reports the max time over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

M_TOK, K_IN, N_OUT, BLOCK = 12000, 5376, 7168, 128
GEMM_OPS = 2 * M_TOK * N_OUT * K_IN          # one GEMM launch
STEP_OPS = 3 * GEMM_OPS                       # fwd + dX + dW
UPDATE_BYTES = 22 * N_OUT * K_IN              # AdamW SR update: 1+4+4+4 in, 1+4+4 out
METRIC = "INT8 qlinear fwd+bwd TOPS (3 int8 GEMMs per train step of the 5376->7168 layer, 12000 tokens)"
WORKLOAD = ("qlinear train step: M=12000 K=5376 N=7168, Hadamard block 128, bf16 X/dY/y/dX, "
            "fwd + dX + dW + AdamW stochastic requant")
NOMINAL_INT8_OVER_BF16 = 2.0   # dense int8 4.5 POPS / dense bf16 2.25 PFLOPS
NOMINAL_INT8_TOPS = 4500.0     # B200 dense int8 spec, for context next to the measured proxy

# DRAM bytes (read + write) per GEMM launch from an ncu capture of the
# 12000-token layer step (mean of the forward, input-gradient and
# weight-gradient launches), valid only for the GEMM source it was taken on.
GEMM_TRAFFIC_BYTES = 336.2e6
GEMM_TRAFFIC_SOURCE_SHA = "99e20f7e2ee73977"
# The same for the update kernel on the [7168, 5376] weight; DRAM writes
# still held in L2 when the kernel ends are not counted.
UPDATE_TRAFFIC_BYTES = 790.6e6
UPDATE_TRAFFIC_SOURCE_SHA = "af301d8b5fe11a46"


def source_sha(files=("gemm_i8.cu", "sm100.cuh")):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "int8_quantized_act_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gemm_source_sha():
    return source_sha()


UPDATE_SOURCES = ("update_sr.cu", "rowops.cuh", "divrn.cuh", "sm100.cuh")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--e2e-steps", type=int, default=60)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--routes", action="store_true",
                   help="instead of the train step: time the forward's int8 and bf16 routes "
                        "at 2048 and 12000 tokens (one JSON line)")
    p.add_argument("--swiglu", action="store_true",
                   help="instead of the train step: one SwiGLU MLP training step (d_model 4096, "
                        "d_ff 14336, 8192 tokens; one JSON line)")
    p.add_argument("--sweep", action="store_true",
                   help="instead of the train step: the AdamW stochastic-requant update (plain and "
                        "row-wise weight norm) on [n, n] weights, n = 1024 .. 16384 (one JSON line)")
    p.add_argument("--kernel", default=None,
                   help="instead of the train step: time one library call of a single kernel "
                        "family at its full-size shape (quant, quant_dy, bwd, update_staged, "
                        "update_rows, update_wn, update_wn16, gate, gate_bwd, bf16gemm, muon)")
    p.add_argument("--muon", action="store_true",
                   help="instead of the train step: one MuonAuxAdamW step of the 5376->7168 weight "
                        "(one JSON line)")
    p.add_argument("--edge", action="store_true",
                   help="instead of the train step: time the layer's calls at 1..128 tokens, "
                        "where the weight stream bounds the forward (one JSON line)")
    return p.parse_args()


# ---------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank number over all ranks (NCCL on the GPUs; gloo on CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(world, steps, ms_max):
    """Whole-job throughput: each of `world` replicas runs `steps` full layer
    steps; the job takes the slowest rank's time."""
    return world * STEP_OPS * steps / (ms_max * 1e-3) / 1e12


# ---------------------------------------------------------------- peaks / clocks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- our path
class Layer:
    """Device state of one replica: the prepared int8 weight, AdamW moments,
    bf16 X / dY of one batch, outputs and the backward workspace."""

    def __init__(self):
        import torch
        import int8_quantized_act_b200 as ql
        import workloads
        self.ql, self.torch = ql, torch
        d = workloads.rotated_layer(M=M_TOK, seed=1)
        dev = "cuda"
        self.x_host = d["x_bf16"].pin_memory()
        self.dy_host = d["dy_bf16"].pin_memory()
        self.x = self.x_host.to(dev)
        self.dy = self.dy_host.to(dev)
        self.bias = torch.from_numpy(d["bias"]).to(dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.wq = torch.empty((N_OUT, K_IN), dtype=torch.int8, device=dev)
        self.sw = torch.empty(N_OUT, dtype=torch.float32, device=dev)
        ql.qlinear_quantize_rows(torch.from_numpy(d["w"]).to(dev), self.wq, self.sw, self.status,
                                 hadamard_block=BLOCK, flags=ql.QL_REJECT_ZERO_ROWS)
        self.m = torch.zeros((N_OUT, K_IN), dtype=torch.float32, device=dev)
        self.v = torch.zeros((N_OUT, K_IN), dtype=torch.float32, device=dev)
        self.y = torch.empty((M_TOK, N_OUT), dtype=torch.bfloat16, device=dev)
        self.xq = torch.empty((M_TOK, K_IN), dtype=torch.int8, device=dev)
        self.sx = torch.empty(M_TOK, dtype=torch.float32, device=dev)
        self.dx = torch.empty((M_TOK, K_IN), dtype=torch.bfloat16, device=dev)
        self.dw = torch.empty((N_OUT, K_IN), dtype=torch.float32, device=dev)
        self.db = torch.empty(N_OUT, dtype=torch.float32, device=dev)
        self.ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M_TOK, N_OUT, K_IN, BLOCK),
                              dtype=torch.uint8, device=dev)
        self.opt = ql.Optim(kind=ql.QL_ADAMW, lr=1e-3, weight_decay=0.01)
        self.t = 0
        # the step's result read back by the end-to-end loop: the status word
        # and the bias gradient (y and dX stay on the device, for the layers
        # next to this one)
        self.status_host = torch.empty(1, dtype=torch.int32).pin_memory()
        self.db_host = torch.empty(N_OUT, dtype=torch.float32).pin_memory()
        torch.cuda.synchronize()

    def step(self, gemm_events=None, update_events=None, bufs=None):
        ql = self.ql
        self.t += 1
        x, dy, y, dx = bufs or (self.x, self.dy, self.y, self.dx)
        # events around the forward, input-gradient and weight-gradient GEMMs
        # and (update_events) around the forward call, the backward call and
        # the update
        ql.ql_set_gemm_timing_events(gemm_events or ())
        if update_events:
            update_events[2].record()
        ql.qlinear_fwd(x, self.wq, self.sw, self.bias, BLOCK, y, self.xq, self.sx, self.status)
        if update_events:
            update_events[3].record()
        ql.qlinear_bwd(dy, self.wq, self.sw, self.xq, self.sx, BLOCK, dx, self.dw, self.db,
                       self.ws, self.status)
        ql.ql_set_gemm_timing_events(())
        if update_events:
            update_events[0].record()
        ql.qweight_update_sr(self.wq, self.sw, self.dw, self.opt, self.m, self.v, 1234, self.t,
                             self.status)
        if update_events:
            update_events[1].record()

    def copy_floor(self, reps=5):
        """Device time of one step's copies alone: X and dY in from the pinned
        host buffers, then the result out (the PCIe bound of run_e2e)."""
        torch = self.torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def once():
            self.x.copy_(self.x_host, non_blocking=True)
            self.dy.copy_(self.dy_host, non_blocking=True)
            self.db_host.copy_(self.db, non_blocking=True)
            self.status_host.copy_(self.status, non_blocking=True)

        once()
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            once()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    def run_e2e(self, steps):
        """`steps` layer steps through the public API with host buffers: each
        step copies its X and dY in from pinned host memory and reads its
        result back (the status word and the bias gradient).  The copies in
        run on their own stream into two buffer sets, so step i+1's inputs
        cross PCIe while step i computes, the way a training loop overlaps
        data movement.  Returns the device time from the first copy in to
        the last read-back."""
        torch = self.torch
        if not hasattr(self, "bufs"):
            self.bufs = [(self.x, self.dy), (torch.empty_like(self.x), torch.empty_like(self.dy))]
            self.s_in, self.s_comp = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for s in (self.s_in, self.s_comp):
            s.wait_event(start)
        in_done, comp_done = {}, {}
        for i in range(steps):
            x, dy = self.bufs[i % 2]
            with torch.cuda.stream(self.s_in):
                if i >= 2:
                    self.s_in.wait_event(comp_done[i - 2])  # step i-2 is done reading x, dy
                x.copy_(self.x_host, non_blocking=True)
                dy.copy_(self.dy_host, non_blocking=True)
                in_done[i] = ev()
                in_done[i].record()
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(in_done[i])
                self.step(bufs=(x, dy, self.y, self.dx))
                self.db_host.copy_(self.db, non_blocking=True)
                self.status_host.copy_(self.status, non_blocking=True)
                comp_done[i] = ev()
                comp_done[i].record()
        cur = torch.cuda.current_stream()
        cur.wait_stream(self.s_comp)
        cur.wait_stream(self.s_in)
        stop.record()
        torch.cuda.synchronize()
        return start.elapsed_time(stop)


def new_events(n):
    import torch
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()  # materialise the CUDA event before the library records it
    return evs


def run_ours(args, rank, world, local):
    import torch
    import int8_quantized_act_b200 as ql

    layer = Layer()
    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    gemm_ev = [list(zip(*[iter(new_events(6))] * 2)) for _ in range(args.steps)]
    upd_ev = [new_events(4) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = ql.ql_kernel_launches()
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    barrier(world)
    clocks.start()
    time.sleep(0.2)  # let the sampler start before the timed region
    torch.cuda.synchronize()
    start.record()
    for i in range(args.steps):
        layer.step(gemm_ev[i], upd_ev[i])
    stop.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    launches = ql.ql_kernel_launches() - launches0
    ms = start.elapsed_time(stop)
    ms_max = max_over_ranks(ms, world)
    word = int(layer.status.item())
    if word:
        raise RuntimeError(f"device status {ql.status_flags(word)}")

    gemm_ms = [b.elapsed_time(a) for pairs in gemm_ev for (b, a) in pairs]
    per_kind = {name: statistics.mean(gemm_ms[j::3]) for j, name in enumerate(("fwd", "dx", "dw"))}
    gemm_avg = statistics.mean(gemm_ms)
    upd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in upd_ev)
    fwd_call_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in upd_ev)
    bwd_call_ms = statistics.mean(e[3].elapsed_time(e[0]) for e in upd_ev)

    # end to end through the public API with host buffers
    e2e_steps = max(2, min(args.e2e_steps, args.steps))
    layer.run_e2e(2)
    barrier(world)
    e2e_ms = max_over_ranks(layer.run_e2e(e2e_steps), world) / e2e_steps
    copy_ms = layer.copy_floor()
    word = int(layer.status.item())
    if word:
        raise RuntimeError(f"device status {ql.status_flags(word)}")

    peaks = load_peaks()
    int8_peak = peaks["bf16_tflops"] * NOMINAL_INT8_OVER_BF16
    gemm_tops = GEMM_OPS / (gemm_avg * 1e-3) / 1e12
    value = job_tops(world, args.steps, ms_max)
    h2d = layer.x.numel() * 2 + layer.dy.numel() * 2
    d2h = layer.db_host.numel() * 4 + layer.status_host.numel() * 4
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "i8",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_TOK, "K": K_IN, "N": N_OUT,
                   "hadamard_block": BLOCK, "x_dtype": "bf16", "dy_dtype": "bf16",
                   "y_dtype": "bf16", "dx_dtype": "bf16", "dw_dtype": "f32",
                   "optimizer": "AdamW lr=1e-3 wd=0.01, fp32 moments",
                   "l2": "no flush: step working set ~1.1 GB > 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "gemm_i8 (tcgen05 kind::i8, fwd/dX/dW launches)",
                     "achieved": round(gemm_tops, 1),
                     "peak": round(int8_peak, 1), "unit": "TOPS",
                     "frac": round(gemm_tops / int8_peak, 4),
                     "peak_source": f"{peaks['source']}: bf16 dense burst x {NOMINAL_INT8_OVER_BF16} (int8/bf16 nominal ratio)",
                     "ms_per_launch": {k: round(v, 4) for k, v in per_kind.items()},
                     "traffic": (GEMM_TRAFFIC_BYTES if gemm_source_sha() == GEMM_TRAFFIC_SOURCE_SHA
                                 else None),
                     "traffic_unit": "bytes per launch",
                     "frac_of_nominal_int8": round(gemm_tops / NOMINAL_INT8_TOPS, 4),
                     # the same against the sustained (power-capped, seconds-long) bf16 figure,
                     # and against the burst peak scaled to the median SM clock sampled in the
                     # timed region
                     "frac_of_sustained": round(gemm_tops / (peaks["bf16_tflops_sustained"]
                                                              * NOMINAL_INT8_OVER_BF16), 4),
                     "frac_at_sampled_clock": (round(gemm_tops / (int8_peak * clk["sm_mhz"]
                                                                  / clk["sm_max_mhz"]), 4)
                                               if clk.get("sm_mhz") and clk.get("sm_max_mhz")
                                               else None)},
        "row_kernel": {"kernel": "update_sr (AdamW + stochastic requant)", "bound": "hbm",
                       "achieved": round(UPDATE_BYTES / (upd_ms * 1e-3) / 1e9, 1),
                       "peak": peaks["hbm_gbs"], "unit": "GB/s",
                       "frac": round(UPDATE_BYTES / (upd_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                       "ms_per_launch": round(upd_ms, 4),
                       "traffic": (UPDATE_TRAFFIC_BYTES if source_sha(UPDATE_SOURCES) == UPDATE_TRAFFIC_SOURCE_SHA
                                   else None),
                       "traffic_unit": "bytes per launch"},
        "row_kernels_gbs": {
            "note": "algorithmic bytes / call time minus its GEMM launches (so including launch "
                    "gaps): X quantization 3 B/elem; gradient preparation 2 reads of bf16 dY + "
                    "2 int8 code writes = 6 B/elem; update 22 B/elem",
            "quantize_x": round(3 * M_TOK * K_IN / ((fwd_call_ms - per_kind["fwd"]) * 1e-3) / 1e9, 1),
            "gradient_prep": round(6 * M_TOK * N_OUT / ((bwd_call_ms - per_kind["dx"] - per_kind["dw"]) * 1e-3) / 1e9, 1),
            "update": round(UPDATE_BYTES / (upd_ms * 1e-3) / 1e9, 1),
            "peak": peaks["hbm_gbs"],
        },
        "breakdown_ms": {
            "fwd_call": round(fwd_call_ms, 4),
            "fwd_quantize_x": round(fwd_call_ms - per_kind["fwd"], 4),
            "bwd_call": round(bwd_call_ms, 4),
            "bwd_gradient_prep": round(bwd_call_ms - per_kind["dx"] - per_kind["dw"], 4),
            "update": round(upd_ms, 4),
            "note": "CUDA events on the step's stream; fwd_quantize_x and bwd_gradient_prep are "
                    "the call times minus their GEMM launches",
        },
        "e2e": {"value": round(job_tops(world, 1, e2e_ms), 2), "unit": "TOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "overlap": "copies in on their own stream into two buffer sets; the step's "
                           "result (status word, bias gradient) read back after each step",
                "copies_alone_ms": round(copy_ms, 4)},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(seconds=10.0)
    return out


# ---------------------------------------------------------------- CPU oracle
def cpu_sample_step(d, xq_all, sx_all, wq, sw, rows, wcols, urows, t):
    """One bounded sample of the step on the oracle: forward and dX of `rows`
    tokens, dW of `wcols` output rows over all tokens, AdamW requant of
    `urows` weight rows.  Returns the int8 GEMM ops done."""
    import numpy as np
    import oracle
    x = d["x"][:rows]
    oracle.fwd(x, wq, sw, d["bias"], BLOCK)
    oracle.bwd_dx(d["dy"][:rows], wq, sw, BLOCK)
    dw, *_ = oracle.bwd_dw(d["dy"][:, :wcols], xq_all, sx_all)
    g = np.ascontiguousarray(dw[:urows]) if urows <= wcols else np.zeros((urows, K_IN), np.float32)
    zeros = np.zeros((urows, K_IN), np.float32)
    oracle.update_sr(wq[:urows], sw[:urows], g, oracle.ADAMW, 1e-3, 1234, t, m=zeros, v=zeros,
                     wd=0.01)
    return 2 * rows * N_OUT * K_IN * 2 + 2 * wcols * K_IN * M_TOK


def cpu_prepare():
    import oracle
    import workloads
    d = workloads.rotated_layer(M=M_TOK, seed=1)
    wq, sw, _ = oracle.quantize_rows(d["w"], B=BLOCK, flags=oracle.REJECT_ZERO_ROWS)
    xq, sx, _ = oracle.quantize_rows(d["x"], B=BLOCK)
    return d, xq, sx, wq, sw


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---- the oracle on every host core: one single-threaded sample per process
_CPU_ARRAYS = None


def _cpu_worker_init(paths):
    global _CPU_ARRAYS
    import numpy as np
    _CPU_ARRAYS = {k: np.load(v, mmap_mode="r") for k, v in paths.items()}


def _cpu_worker_sample(args):
    """Worker i's sample of step t: forward and dX of 4 tokens, dW of 2
    output rows over all tokens, AdamW requant of 8 weight rows (its own rows
    and columns of the workload).  Returns the int8 GEMM ops done."""
    import numpy as np
    import oracle
    i, t = args
    A = _CPU_ARRAYS
    rows, wcols, urows = 4, 2, 8
    r0 = (i * rows) % (M_TOK - rows)
    c0 = (i * wcols) % (N_OUT - wcols)
    u0 = (i * urows) % (N_OUT - urows)
    oracle.fwd(A["x"][r0:r0 + rows], A["wq"], A["sw"], A["bias"], BLOCK)
    oracle.bwd_dx(A["dy"][r0:r0 + rows], A["wq"], A["sw"], BLOCK)
    dw, *_ = oracle.bwd_dw(np.ascontiguousarray(A["dy"][:, c0:c0 + wcols]), A["xq"], A["sx"])
    g = np.zeros((urows, K_IN), np.float32)
    g[:wcols] = dw
    zeros = np.zeros((urows, K_IN), np.float32)
    oracle.update_sr(A["wq"][u0:u0 + urows], A["sw"][u0:u0 + urows], g, oracle.ADAMW, 1e-3,
                     1234, t, m=zeros, v=zeros, wd=0.01)
    return 2 * rows * N_OUT * K_IN * 2 + 2 * wcols * K_IN * M_TOK


class CpuPool:
    """A process pool (started with spawn, never forked from a process that
    may hold a GPU context) running the oracle as it stands, one sample per
    process per step, on every core of the host."""

    def __init__(self, prepared, cores=None):
        import multiprocessing as mp
        import tempfile
        import numpy as np
        d, xq, sx, wq, sw = prepared
        self.dir = tempfile.mkdtemp(prefix="qlinear_oracle_")
        arrays = {"x": d["x"], "dy": d["dy"], "bias": d["bias"], "xq": xq, "sx": sx, "wq": wq,
                  "sw": sw}
        paths = {}
        for k, v in arrays.items():
            paths[k] = os.path.join(self.dir, k + ".npy")
            np.save(paths[k], np.ascontiguousarray(v))
        self.cores = cores or host_cores()
        self.pool = mp.get_context("spawn").Pool(self.cores, initializer=_cpu_worker_init,
                                                 initargs=(paths,))

    def step(self, t):
        return sum(self.pool.map(_cpu_worker_sample, [(i, t) for i in range(self.cores)],
                                 chunksize=1))

    def close(self):
        import shutil
        self.pool.close()
        self.pool.join()
        shutil.rmtree(self.dir, ignore_errors=True)


def cpu_baseline(seconds=10.0, prepared=None):
    """The oracle as it stands (single-threaded C) on bounded samples of the
    workload, scaled to the metric's unit: on one core, and on every core of
    the host at once (independent samples in a process pool)."""
    prepared = prepared or cpu_prepare()
    d, xq, sx, wq, sw = prepared
    rows, wcols, urows = 4, 2, 8
    ops, t0, t = 0, time.perf_counter(), 0
    while time.perf_counter() - t0 < seconds:
        t += 1
        ops += cpu_sample_step(d, xq, sx, wq, sw, rows, wcols, urows, t)
    el = time.perf_counter() - t0
    single = {"value": round(ops / el / 1e12, 6), "unit": "TOPS", "cores": 1,
              "sample": (f"{t} samples of the step: fwd + dX of {rows} of 12000 tokens, dW of "
                         f"{wcols} of 7168 output rows over all tokens, AdamW requant of {urows} "
                         f"weight rows; {el:.1f} s on one core; ops = int8 GEMM ops done")}
    out = {"value": single["value"], "unit": "TOPS", "cores": 1, "kind": "oracle",
           "cpu_model": cpu_model(), "host_cores": host_cores(), "sample": single["sample"]}
    try:
        pool = CpuPool(prepared)
    except Exception as e:  # no process pool on this host: one core only
        out["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
        return out
    try:
        pool.step(0)  # warm-up: workers import and map the arrays
        mops, t0, steps = 0, time.perf_counter(), 0
        while time.perf_counter() - t0 < seconds:
            steps += 1
            mops += pool.step(steps)
        mel = time.perf_counter() - t0
    finally:
        pool.close()
    out.update({"value": round(mops / mel / 1e12, 6), "cores": pool.cores,
                "sample": (f"{steps} rounds of {pool.cores} concurrent single-threaded samples "
                           f"(one per core; each as below, on its own rows and columns) in "
                           f"{mel:.1f} s"),
                "single_thread": single})
    return out


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands on every host core, each
    step one bounded sample per core (rank 0 only; other ranks exit)."""
    if rank != 0:
        return None
    prepared = cpu_prepare()
    pool = CpuPool(prepared)
    try:
        for i in range(max(1, args.warmup)):
            pool.step(i + 1)
        ops, t0 = 0, time.perf_counter()
        for i in range(args.steps):
            ops += pool.step(i + 1)
        el = time.perf_counter() - t0
    finally:
        pool.close()
    value = ops / el / 1e12
    sample = (f"each step: one sample per core on {pool.cores} cores, each fwd + dX of 4 of "
              f"12000 tokens, dW of 2 of 7168 output rows over all tokens, AdamW requant of 8 "
              f"weight rows")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M_TOK, "K": K_IN, "N": N_OUT,
                   "hadamard_block": BLOCK, "parallelism": "cpu oracle, rank 0, all host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": pool.cores,
                         "kind": "oracle", "cpu_model": cpu_model(), "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_routes(args):
    """The page's forward-route comparison on this GPU: the int8 route
    (rotate + quantize x, int8 GEMM) against the bf16 route (rotate x to
    bf16, bf16 GEMM against the codes as bf16, converted once per weight
    update and timed separately) at 2048 and 12000 tokens of the 5376 ->
    7168 layer, block 128, bf16 x and y.  Whole-call and GEMM-only device
    times (CUDA events), medians over `steps` calls."""
    import torch
    import int8_quantized_act_b200 as ql
    import workloads
    torch.cuda.set_device(0)
    peaks = load_peaks()
    out = {"metric": "forward route time (ms per call)", "unit": "ms", "higher_is_better": False,
           "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "data": "synthetic",
           "config": {"workload": "5376 -> 7168 layer forward, Hadamard block 128, bf16 x and y",
                      "K": K_IN, "N": N_OUT, "hadamard_block": BLOCK},
           "routes": {}}
    d = workloads.rotated_layer(M=12000, seed=1)
    dev = "cuda"
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    wq = torch.empty((N_OUT, K_IN), dtype=torch.int8, device=dev)
    sw = torch.empty(N_OUT, device=dev)
    ql.qlinear_quantize_rows(torch.from_numpy(d["w"]).to(dev), wq, sw, st, hadamard_block=BLOCK,
                             flags=ql.QL_REJECT_ZERO_ROWS)
    wb = torch.empty((N_OUT, K_IN), dtype=torch.bfloat16, device=dev)
    bias = torch.from_numpy(d["bias"]).to(dev)
    x_all = d["x_bf16"].to(dev)

    def timed(fn, gemm=False):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        gev = [tuple(new_events(2)) for _ in range(args.steps)] if gemm else None
        for _ in range(args.warmup):
            fn(None)
        torch.cuda.synchronize()
        for i in range(args.steps):
            ev[i][0].record()
            fn(gev[i] if gemm else None)
            ev[i][1].record()
        torch.cuda.synchronize()
        call = statistics.median(a.elapsed_time(b) for a, b in ev)
        g = statistics.median(a.elapsed_time(b) for a, b in gev) if gemm else None
        return call, g

    ms_codes, _ = timed(lambda _e: ql.qlinear_codes_bf16(wq, wb))
    out["codes_bf16_ms"] = round(ms_codes, 4)
    for M in (2048, 12000):
        x = x_all[:M].contiguous()
        y = torch.empty((M, N_OUT), dtype=torch.bfloat16, device=dev)
        xq = torch.empty((M, K_IN), dtype=torch.int8, device=dev)
        sx = torch.empty(M, device=dev)
        ws = torch.empty(ql.qlinear_fwd_bf16_workspace_bytes(M, K_IN, torch.bfloat16, BLOCK),
                         dtype=torch.uint8, device=dev)

        def int8_route(g):
            ql.ql_set_gemm_timing_events([g] if g else ())
            ql.qlinear_fwd(x, wq, sw, bias, BLOCK, y, xq, sx, st)
            ql.ql_set_gemm_timing_events(())

        def bf16_route(g):
            ql.ql_set_gemm_timing_events([g] if g else ())
            ql.qlinear_fwd_bf16(x, wb, sw, bias, BLOCK, y, ws, st)
            ql.ql_set_gemm_timing_events(())

        ops = 2.0 * M * N_OUT * K_IN
        c8, g8 = timed(int8_route, gemm=True)
        cb, gb = timed(bf16_route, gemm=True)
        out["routes"][str(M)] = {
            "int8_ms": round(c8, 4), "int8_gemm_ms": round(g8, 4),
            "int8_gemm_tops": round(ops / (g8 * 1e-3) / 1e12, 1),
            "bf16_ms": round(cb, 4), "bf16_gemm_ms": round(gb, 4),
            "bf16_gemm_tflops": round(ops / (gb * 1e-3) / 1e12, 1),
            "bf16_gemm_frac_of_measured_bf16_peak": round(ops / (gb * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
        }
    if int(st.item()):
        raise RuntimeError(f"device status {ql.status_flags(int(st.item()))}")
    return out


def run_edge(args):
    """The 5376 -> 7168 layer (block 128, bf16) at 1, 4, 15, 16, 17, 64 and 128
    tokens: forward, input gradient and weight gradient, whole call and GEMM
    alone (CUDA events around single calls, medians; these include the host's
    launch latency), and the device time per call with 20 calls captured in
    a CUDA graph.  Below a GEMM's row floor the forward reads the 38.5 MB int8
    weight once per call, so its bound is that read."""
    import torch
    import int8_quantized_act_b200 as ql
    import workloads
    torch.cuda.set_device(0)
    peaks = load_peaks()
    d = workloads.rotated_layer(M=128, seed=1)
    dev = "cuda"
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    wq = torch.empty((N_OUT, K_IN), dtype=torch.int8, device=dev)
    sw = torch.empty(N_OUT, device=dev)
    ql.qlinear_quantize_rows(torch.from_numpy(d["w"]).to(dev), wq, sw, st, hadamard_block=BLOCK,
                             flags=ql.QL_REJECT_ZERO_ROWS)
    bias = torch.from_numpy(d["bias"]).to(dev)
    x_all, dy_all = d["x_bf16"].to(dev), d["dy_bf16"].to(dev)
    w_bytes = N_OUT * K_IN
    out = {"metric": "layer call time at small token counts (us per call)", "unit": "us",
           "higher_is_better": False, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
           "data": "synthetic",
           "config": {"workload": "5376 -> 7168 layer, Hadamard block 128, bf16 x, dY, y, dX",
                      "K": K_IN, "N": N_OUT, "weight_bytes": w_bytes,
                      "hbm_peak_gbs": peaks["hbm_gbs"]},
           "tokens": {}}

    def timed(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        gev = [tuple(new_events(2)) for _ in range(args.steps)]
        for _ in range(args.warmup):
            fn(None)
        torch.cuda.synchronize()
        for i in range(args.steps):
            ev[i][0].record()
            fn(gev[i])
            ev[i][1].record()
        torch.cuda.synchronize()
        return (statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3,
                statistics.median(a.elapsed_time(b) for a, b in gev) * 1e3)

    def graph_us(call, reps=20):
        """Device time per call with the host out of the way: `reps` calls
        captured in one CUDA graph, replayed after a warm-up."""
        call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                call()
        for _ in range(args.warmup):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(args.steps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1e3 / (args.steps * reps)

    for M in (1, 4, 15, 16, 17, 64, 128):
        x, dy = x_all[:M].contiguous(), dy_all[:M].contiguous()
        y = torch.empty((M, N_OUT), dtype=torch.bfloat16, device=dev)
        xq = torch.empty((M, K_IN), dtype=torch.int8, device=dev)
        sx = torch.empty(M, device=dev)
        dx = torch.empty((M, K_IN), dtype=torch.bfloat16, device=dev)
        dw = torch.empty((N_OUT, K_IN), device=dev)
        db = torch.empty(N_OUT, device=dev)
        ws = torch.empty(ql.qlinear_workspace_bytes(M, N_OUT, K_IN, BLOCK), dtype=torch.uint8,
                         device=dev)

        def with_events(call):
            def f(g):
                ql.ql_set_gemm_timing_events([g] if g else ())
                call()
                ql.ql_set_gemm_timing_events(())
            return f

        calls = {
            "fwd": lambda: ql.qlinear_fwd(x, wq, sw, bias, BLOCK, y, xq, sx, st),
            "dx": lambda: ql.qlinear_bwd_dx(dy, wq, sw, BLOCK, dx, ws, st),
            "dw": lambda: ql.qlinear_bwd_dw(dy, xq, sx, dw, db, ws, st),
        }
        row = {}
        for name, call in calls.items():
            t_call, t_gemm = timed(with_events(call))
            row[f"{name}_us"] = round(t_call, 2)
            row[f"{name}_gemm_us"] = round(t_gemm, 2)
            row[f"{name}_graph_us"] = round(graph_us(call), 2)
        row["fwd_graph_weight_gbs"] = round(w_bytes / (row["fwd_graph_us"] * 1e-6) / 1e9, 1)
        row["dx_graph_weight_gbs"] = round(w_bytes / (row["dx_graph_us"] * 1e-6) / 1e9, 1)
        row["dw_graph_output_gbs"] = round(4 * w_bytes / (row["dw_graph_us"] * 1e-6) / 1e9, 1)
        out["tokens"][str(M)] = row
    if int(st.item()):
        raise RuntimeError(f"device status {ql.status_flags(int(st.item()))}")
    return out


def run_swiglu(args):
    """A SwiGLU MLP training step through the library's calls: d_model 4096,
    d_ff 14336, 8192 tokens, bf16 activations and gradients, no rotation,
    AdamW (lr 1e-3, wd 0.01) with stochastic requantization of both weights.
    w1 and w3 run stacked as one [28672, 4096] weight (one quantization of X
    for both); the gate h = silu(a) * b runs fused with the quantization of
    the second projection's input (qlinear_swiglu_quantize, h never stored),
    the second projection takes those codes (qlinear_fwd_quantized), and the
    gate's backward (qlinear_swiglu_bwd) gives the stacked projection's
    output gradient.  Every step of it is one of the library's kernels.
    Metric: the 9 int8 GEMMs' operations (3 x 2 x 8192 x 4096 x 14336 x 3)
    per second of the whole step."""
    import torch
    import int8_quantized_act_b200 as ql
    torch.cuda.set_device(0)
    T, D, F = 8192, 4096, 14336
    gen = torch.Generator(device="cuda").manual_seed(5)
    dev = "cuda"

    def normal(shape, std, dtype=torch.float32):
        return (torch.randn(shape, generator=gen, device=dev) * std).to(dtype)

    st = torch.zeros(1, dtype=torch.int32, device=dev)

    class Weight:
        def __init__(self, n, k):
            self.q = torch.empty((n, k), dtype=torch.int8, device=dev)
            self.s = torch.empty(n, device=dev)
            ql.qlinear_quantize_rows(normal((n, k), 0.02), self.q, self.s, st,
                                     flags=ql.QL_REJECT_ZERO_ROWS)
            self.m = torch.zeros((n, k), device=dev)
            self.v = torch.zeros((n, k), device=dev)
            self.dw = torch.empty((n, k), device=dev)
            self.db = torch.empty(n, device=dev)

    w13, w2 = Weight(2 * F, D), Weight(D, F)
    x = normal((T, D), 1.0, torch.bfloat16)
    dy = normal((T, D), 1.0, torch.bfloat16)
    h13 = torch.empty((T, 2 * F), dtype=torch.bfloat16, device=dev)
    xq = torch.empty((T, D), dtype=torch.int8, device=dev)
    sx = torch.empty(T, device=dev)
    hq = torch.empty((T, F), dtype=torch.int8, device=dev)
    sh = torch.empty(T, device=dev)
    y = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    dh = torch.empty((T, F), dtype=torch.bfloat16, device=dev)
    d13 = torch.empty((T, 2 * F), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(ql.qlinear_bwd_workspace_bytes(T, D, F, 0),
                         ql.qlinear_bwd_workspace_bytes(T, 2 * F, D, 0)), dtype=torch.uint8,
                     device=dev)
    opt = ql.Optim(kind=ql.QL_ADAMW, lr=1e-3, weight_decay=0.01)
    t = [0]

    def step(ev=None):
        t[0] += 1
        rec = (lambda i: ev[i].record()) if ev else (lambda i: None)
        rec(0)
        ql.qlinear_fwd(x, w13.q, w13.s, None, 0, h13, xq, sx, st)
        rec(1)
        ql.qlinear_swiglu_quantize(h13, hq, sh, st)
        rec(2)
        ql.qlinear_fwd_quantized(hq, sh, w2.q, w2.s, None, y, st)
        ql.qlinear_bwd(dy, w2.q, w2.s, hq, sh, 0, dh, w2.dw, w2.db, ws, st)
        rec(3)
        ql.qlinear_swiglu_bwd(h13, dh, d13)
        rec(4)
        ql.qlinear_bwd(d13, w13.q, w13.s, xq, sx, 0, dx, w13.dw, w13.db, ws, st)
        rec(5)
        ql.qweight_update_sr(w13.q, w13.s, w13.dw, opt, w13.m, w13.v, 11, t[0], st)
        ql.qweight_update_sr(w2.q, w2.s, w2.dw, opt, w2.m, w2.v, 12, t[0], st)
        rec(6)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [new_events(7) for _ in range(args.steps)]
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.2)
    torch.cuda.synchronize()
    launches0 = ql.ql_kernel_launches()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    launches = ql.ql_kernel_launches() - launches0
    clk = clocks.stop()
    if int(st.item()):
        raise RuntimeError(f"device status {ql.status_flags(int(st.item()))}")
    el = lambda i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in evs)
    step_ms = el(0, 6)
    gate_ms, gate_bwd_ms = el(1, 2), el(3, 4)
    upd_ms = el(5, 6)
    ops = 9 * 2.0 * T * D * F
    upd_bytes = 22 * (2 * F * D + D * F)
    # the gate reads bf16 [a | b] and writes int8 h codes; its backward reads
    # [a | b] and dh and writes [da | db], all bf16
    gate_bytes = T * F * (4 + 1)
    gate_bwd_bytes = T * F * (4 + 2 + 4)
    peaks = load_peaks()
    return {
        "metric": "SwiGLU MLP train step TOPS (9 int8 GEMMs per step, d_model 4096, d_ff 14336, 8192 tokens)",
        "value": round(ops / (step_ms * 1e-3) / 1e12, 2), "unit": "TOPS", "higher_is_better": True,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "data": "synthetic",
        "dtype": "i8",
        "config": {"workload": "SwiGLU MLP step: w1|w3 stacked [28672,4096], w2 [4096,14336], "
                               "8192 tokens, bf16 x/dY, fused gate + h quantization, AdamW + "
                               "stochastic requant of both weights",
                   "tokens": T, "d_model": D, "d_ff": F},
        "ms_per_step": round(step_ms, 4),
        "gpu_launches": launches,
        "breakdown_ms": {"gate_fwd_quant": round(gate_ms, 4), "gate_bwd": round(gate_bwd_ms, 4),
                         "updates": round(upd_ms, 4)},
        "gate_fwd_gbs": round(gate_bytes / (gate_ms * 1e-3) / 1e9, 1),
        "gate_bwd_gbs": round(gate_bwd_bytes / (gate_bwd_ms * 1e-3) / 1e9, 1),
        "update_gbs": round(upd_bytes / (upd_ms * 1e-3) / 1e9, 1),
        "update_frac_of_hbm": round(upd_bytes / (upd_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "clocks": clk,
    }


def run_sweep(args):
    """The update on square weights n x n, n = 1024, 2048, 4096, 8192, 16384:
    AdamW (lr 1e-3, wd 0.01) with stochastic requantization, plain and with
    the row-wise weight norm (float32 magnitude per row and its moments).
    Bytes per call: 22 per element (codes 1 + gradient 4 + moments 8 in; codes
    1 + moments 8 out) plus, for the weight norm, 24 per row (magnitude and its
    two moments read and written).  Device time per call (CUDA events, median)."""
    import torch
    import int8_quantized_act_b200 as ql
    torch.cuda.set_device(0)
    peaks = load_peaks()
    gen = torch.Generator(device="cuda").manual_seed(9)
    out = {"metric": "AdamW stochastic-requant update bandwidth (GB/s)", "unit": "GB/s",
           "higher_is_better": True, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
           "data": "synthetic", "peak_gbs": peaks["hbm_gbs"],
           "config": {"workload": "update of int8 [n, n] weights, grads ~N(0, 1e-3), AdamW "
                                  "lr 1e-3 wd 0.01, fp32 moments; weight norm: g ~U(0.5, 2)"},
           "sizes": {}}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    opt = ql.Optim(kind=ql.QL_ADAMW, lr=1e-3, weight_decay=0.01)
    for n in (1024, 2048, 4096, 8192, 16384):
        w = torch.randn((n, n), generator=gen, device="cuda") * 0.02
        q = torch.empty((n, n), dtype=torch.int8, device="cuda")
        sw = torch.empty(n, device="cuda")
        ql.qlinear_quantize_rows(w, q, sw, st, flags=ql.QL_REJECT_ZERO_ROWS)
        del w
        g = torch.randn((n, n), generator=gen, device="cuda") * 1e-3
        m = torch.zeros((n, n), device="cuda")
        v = torch.zeros((n, n), device="cuda")
        gm = torch.rand(n, generator=gen, device="cuda") * 1.5 + 0.5
        gmm, gmv = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
        row = {}
        for name, kw in (("adamw", {}), ("adamw_weight_norm", {"g": gm, "g_m": gmm, "g_v": gmv})):
            t = [0]

            def call():
                t[0] += 1
                ql.qweight_update_sr(q, sw, g, opt, m, v, 3, t[0], st, **kw)

            for _ in range(args.warmup):
                call()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            torch.cuda.synchronize()
            for a, b in ev:
                a.record()
                call()
                b.record()
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in ev)
            nbytes = 22 * n * n + (24 * n if kw else 0)
            row[f"{name}_us"] = round(ms * 1e3, 1)
            row[f"{name}_gbs"] = round(nbytes / (ms * 1e-3) / 1e9, 1)
            row[f"{name}_frac"] = round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
        out["sizes"][str(n)] = row
        del q, g, m, v
        torch.cuda.empty_cache()
    if int(st.item()):
        raise RuntimeError(f"device status {ql.status_flags(int(st.item()))}")
    return out


def run_muon(args):
    """One MuonAuxAdamW step of the 5376 -> 7168 layer's int8 weight: Muon
    momentum and five Newton-Schulz steps on the tensor cores (bf16 operands,
    float32 accumulation), then the Muon requantization step; plus AdamW on
    the layer's float bias.  Metric: Newton-Schulz tensor operations per
    second (per step: A = X X^T, A A and B X with X = U^T, r = 5376,
    c = 7168)."""
    import torch
    import int8_quantized_act_b200 as ql
    torch.cuda.set_device(0)
    N, K = N_OUT, K_IN
    r, c = min(N, K), max(N, K)
    gen = torch.Generator(device="cuda").manual_seed(6)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    sw = torch.empty(N, device="cuda")
    ql.qlinear_quantize_rows(torch.randn((N, K), generator=gen, device="cuda") * 0.02, wq, sw, st,
                             flags=ql.QL_REJECT_ZERO_ROWS)
    grad = torch.randn((N, K), generator=gen, device="cuda") * 1e-3
    mom = torch.zeros((N, K), device="cuda")
    O = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(ql.qweight_muon_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    bias = torch.zeros(N, device="cuda")
    gb = torch.randn(N, generator=gen, device="cuda") * 1e-3
    bm, bv = torch.zeros(N, device="cuda"), torch.zeros(N, device="cuda")
    opt = ql.Optim(kind=ql.QL_ADAMW, lr=1e-3, weight_decay=0.0)
    t = [0]

    def step(ev=None):
        t[0] += 1
        rec = (lambda i: ev[i].record()) if ev else (lambda i: None)
        rec(0)
        ql.qweight_muon_orthogonalize(grad, mom, O, ws, st)
        rec(1)
        ql.qweight_update_muon_sr(wq, sw, O, 0.02, 0.01, 13, t[0], st)
        ql.qvector_adamw(bias, gb, bm, bv, opt, t[0], st)
        rec(2)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [new_events(3) for _ in range(args.steps)]
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.2)
    torch.cuda.synchronize()
    launches0 = ql.ql_kernel_launches()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    launches = ql.ql_kernel_launches() - launches0
    clk = clocks.stop()
    if int(st.item()):
        raise RuntimeError(f"device status {ql.status_flags(int(st.item()))}")
    el = lambda i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in evs)
    ns_ms, upd_ms = el(0, 1), el(1, 2)
    # The three products of a Newton-Schulz step as written (X X^T, A A, B X);
    # the two symmetric ones run on their upper 256 x 256 tiles only (the
    # lower tiles are copied), so the tensor cores execute fewer of them.
    ns_ops = 5 * (2.0 * r * r * c + 2.0 * r * r * r + 2.0 * r * c * r)
    nt = (r + 255) // 256
    upper = nt * (nt + 1) / 2 / (nt * nt) if r > 128 else 1.0
    exec_ops = 5 * (upper * (2.0 * r * r * c + 2.0 * r * r * r) + 2.0 * r * c * r)
    peaks = load_peaks()
    tflops = ns_ops / (ns_ms * 1e-3) / 1e12
    exec_tflops = exec_ops / (ns_ms * 1e-3) / 1e12
    upd_bytes = N * K * (1 + 2 + 1)  # codes in, O in (bf16), codes out
    return {
        "metric": "MuonAuxAdamW step of the 5376->7168 weight: Newton-Schulz TFLOP/s",
        "value": round(tflops, 1), "unit": "TFLOP/s", "higher_is_better": True,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "data": "synthetic",
        "dtype": "bf16",
        "config": {"workload": "Muon momentum + 5 Newton-Schulz steps (bf16 tcgen05) + Muon "
                               "stochastic requant of the [7168, 5376] int8 weight + AdamW on its "
                               "bias", "N": N, "K": K},
        "ms_per_step": round(ns_ms + upd_ms, 4), "gpu_launches": launches,
        "breakdown_ms": {"orthogonalize": round(ns_ms, 4), "requant_and_bias": round(upd_ms, 4)},
        "value_note": "the products' FLOPs as written per unit time; the symmetric two run "
                      "on their upper tiles only",
        "executed_tflops": round(exec_tflops, 1),
        "ns_frac_of_bf16_peak": round(exec_tflops / peaks["bf16_tflops"], 4),
        "requant_gbs": round(upd_bytes / (upd_ms * 1e-3) / 1e9, 1),
        "peaks_source": peaks["source"], "clocks": clk,
    }


KERNEL_CASES = {
    # name: (what one call is, algorithmic bytes moved per call)
    "quant": ("qlinear_quantize_rows: 12000 x 5376 bf16 rows, Hadamard block 128", 12000 * 5376 * 3),
    "quant_dy": ("qlinear_quantize_rows: 12000 x 7168 bf16 rows scaled per column (dY * s_w)",
                 12000 * 7168 * 3),
    "bwd": ("qlinear_bwd at 12000 tokens (gradient preparation + both GEMMs)", None),
    "update_staged": ("qweight_update_sr AdamW [7168, 5376]", 22 * 7168 * 5376),
    "update_rows": ("qweight_update_sr AdamW [4096, 14336]", 22 * 4096 * 14336),
    "update_wn": ("qweight_update_sr AdamW + weight norm [8192, 8192]", 22 * 8192 * 8192 + 24 * 8192),
    "update_wn16": ("qweight_update_sr AdamW + weight norm [16384, 16384]",
                    22 * 16384 * 16384 + 24 * 16384),
    "gate": ("qlinear_swiglu_quantize [8192, 2 x 14336] bf16 -> h codes", 8192 * 14336 * 5),
    "gate_bwd": ("qlinear_swiglu_bwd [8192, 2 x 14336] bf16", 8192 * 14336 * 10),
    "bf16gemm": ("qlinear_fwd_bf16 at 12000 tokens (5376 -> 7168, block 128)", None),
    "muon": ("qweight_muon_orthogonalize [7168, 5376]", None),
}


def run_kernel(args):
    """One library call of a single kernel family at its full-size shape,
    timed alone with CUDA events (the shapes the ncu summaries capture)."""
    import torch
    import int8_quantized_act_b200 as ql
    name = args.kernel
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(1)

    def randn(shape, std=1.0, dtype=torch.float32):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(dtype)

    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def wprep(n, k, B=0):
        q = torch.empty((n, k), dtype=torch.int8, device="cuda")
        s = torch.empty(n, device="cuda")
        ql.qlinear_quantize_rows(randn((n, k), 0.02), q, s, st, hadamard_block=B,
                                 flags=ql.QL_REJECT_ZERO_ROWS)
        return q, s

    if name in ("quant", "quant_dy"):
        M, K = (12000, 5376) if name == "quant" else (12000, 7168)
        x = randn((M, K), 1.0, torch.bfloat16)
        q = torch.empty((M, K), dtype=torch.int8, device="cuda")
        s = torch.empty(M, device="cuda")
        cs = randn((K,), 1e-3).abs() + 1e-5 if name == "quant_dy" else None
        B = 128 if name == "quant" else 0

        def run():
            ql.qlinear_quantize_rows(x, q, s, st, col_scale=cs, hadamard_block=B)
    elif name == "bwd":
        M, K, N = M_TOK, K_IN, N_OUT
        wq, sw = wprep(N, K, BLOCK)
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda", generator=g)
        sx = randn((M,), 0.01).abs()
        dy = randn((M, N), 1.0, torch.bfloat16)
        ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M, N, K, BLOCK), dtype=torch.uint8,
                         device="cuda")
        dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        dw = torch.empty((N, K), device="cuda")
        db = torch.empty(N, device="cuda")

        def run():
            ql.qlinear_bwd(dy, wq, sw, xq, sx, BLOCK, dx, dw, db, ws, st)
    elif name.startswith("update"):
        N, K = {"update_rows": (4096, 14336), "update_wn": (8192, 8192),
                "update_wn16": (16384, 16384), "update_staged": (7168, 5376)}[name]
        wq, sw = wprep(N, K)
        grad = randn((N, K), 1e-3)
        m = torch.zeros((N, K), device="cuda")
        v = torch.zeros((N, K), device="cuda")
        wn = None
        if name.startswith("update_wn"):
            wn = (torch.rand(N, generator=g, device="cuda") * 1.5 + 0.5,
                  torch.zeros(N, device="cuda"), torch.zeros(N, device="cuda"))
        opt = ql.Optim(kind=ql.QL_ADAMW, lr=1e-3, weight_decay=0.01)
        step = [0]

        def run():
            step[0] += 1
            if wn is None:
                ql.qweight_update_sr(wq, sw, grad, opt, m, v, 7, step[0], st)
            else:
                ql.qweight_update_sr(wq, sw, grad, opt, m, v, 7, step[0], st, g=wn[0], g_m=wn[1],
                                     g_v=wn[2])
    elif name in ("gate", "gate_bwd"):
        T, F = 8192, 14336
        ab = randn((T, 2 * F), 1.28, torch.bfloat16)
        hq = torch.empty((T, F), dtype=torch.int8, device="cuda")
        sh = torch.empty(T, device="cuda")
        dh = randn((T, F), 1.28, torch.bfloat16)
        dab = torch.empty((T, 2 * F), dtype=torch.bfloat16, device="cuda")

        def run():
            if name == "gate":
                ql.qlinear_swiglu_quantize(ab, hq, sh, st)
            else:
                ql.qlinear_swiglu_bwd(ab, dh, dab)
    elif name == "bf16gemm":
        M, K, N = M_TOK, K_IN, N_OUT
        wq, sw = wprep(N, K, BLOCK)
        wb = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        ql.qlinear_codes_bf16(wq, wb)
        x = randn((M, K), 1.0, torch.bfloat16)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(ql.qlinear_fwd_bf16_workspace_bytes(M, K, torch.bfloat16, BLOCK),
                         dtype=torch.uint8, device="cuda")

        def run():
            ql.qlinear_fwd_bf16(x, wb, sw, None, BLOCK, y, ws, st)
    elif name == "muon":
        N, K = N_OUT, K_IN
        grad = randn((N, K), 1e-3)
        mom = torch.zeros((N, K), device="cuda")
        O = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(ql.qweight_muon_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")

        def run():
            ql.qweight_muon_orthogonalize(grad, mom, O, ws, st)
    else:
        raise SystemExit(f"unknown kernel case {name}; one of {sorted(KERNEL_CASES)}")
    for _ in range(max(1, args.warmup)):
        run()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(args.steps):
        run()
    ev[1].record()
    torch.cuda.synchronize()
    if int(st.item()):
        raise RuntimeError(f"device status {ql.status_flags(int(st.item()))}")
    us = ev[0].elapsed_time(ev[1]) / args.steps * 1e3
    what, nbytes = KERNEL_CASES[name]
    out = {"kernel_case": name, "call": what, "us_per_call": round(us, 2), "calls": args.steps,
           "note": "back-to-back calls, no L2 flush"}
    if nbytes:
        peaks = load_peaks()
        gbs = nbytes / (us * 1e-6) / 1e9
        out.update({"algorithmic_bytes": nbytes, "gbs": round(gbs, 1),
                    "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4), "peaks_source": peaks["source"]})
    return out


def main():
    args = parse_args()
    if args.sweep:
        print(json.dumps(run_sweep(args)), flush=True)
        return
    if args.swiglu:
        print(json.dumps(run_swiglu(args)), flush=True)
        return
    if args.edge:
        print(json.dumps(run_edge(args)), flush=True)
        return
    if args.routes:
        print(json.dumps(run_routes(args)), flush=True)
        return
    if args.muon:
        print(json.dumps(run_muon(args)), flush=True)
        return
    if args.kernel:
        print(json.dumps(run_kernel(args)), flush=True)
        return
    world_env = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, rank, world_env)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        out = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
