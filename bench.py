#!/usr/bin/env python
"""Benchmark of the W4A4 looped quantized linear on B200 (one JSON line).

A step is one pass of the whole hot path over one batch: for each of the T
loops, the fused Kronecker-rotate + group-32 LAS quantizer and the
group-rescaled integer GEMM of every shared linear of the workload
(lq_loop_stack, open mode, weights resident).  Default workload: the
calibration-scale looped block, 7 shared linears (q, k, v, o 2048 x 2048;
gate, up 2048 -> 5632; down 5632 -> 2048) x T = 4 loops on M = 1024 x 256 =
262144 tokens, W4A4, bf16 inputs drawn on the device.  The other workloads
(tiny, the attention projection, the MLP and the decode stacks) are measured
under "aux" with their own TOPS, tokens/s and roofline lines.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lq|reference]
                  [--workload NAME] [--rows M]

With torchrun (N > 1) every rank runs its own replica of the workload on its
GPU (no data-path collective; weak scaling); the time is the max over ranks.
`--impl reference` times the CPU oracle on the host cores instead.
`--rows M` runs the workload with M token rows instead of its own M (the
line's config says so); it exists to profile a full-shape launch on a case
small enough for a detailed capture.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_ptq_looped_b200 import synth  # noqa: E402

DECODE = [synth.decode_workload(M, N, bits) for bits in (8, 4) for N in (2048, 5632)
          for M in (1, 4, 16)]
WORKLOADS = {w.name: w for w in (synth.TINY, synth.ATTN_PROJ, synth.MLP, synth.CALIB_BLOCK,
                                 *DECODE)}
DEFAULT_WORKLOAD = synth.CALIB_BLOCK.name
AUX_WORKLOADS = [synth.TINY.name, synth.ATTN_PROJ.name, synth.MLP.name] + [w.name for w in DECODE]
METRIC = "W4A4 looped-linear TOPS & tokens/s at 1 B200; % of int8 tensor/HBM roofline"
SM_COUNT = 148
SM_CLOCK_GHZ = 1.965
FP64_FMA_PER_SM_CLK = 64  # B200 FP64 units per SM
FP32_LANES_PER_SM = 128  # FP32 FMA lanes per SM
L2_BYTES = 126 << 20
FLUSH_BYTES = 256 << 20


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["lq", "reference"], default="lq")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    p.add_argument("--rows", type=int, default=0, help="token rows M instead of the workload's")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="target CPU time of each oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-probe", action="store_true")
    p.add_argument("--no-aux", action="store_true",
                   help="skip the other workloads and the quantize-only / streaming GEMV lines")
    return p.parse_args()


def workload_of(args):
    wl = WORKLOADS[args.workload]
    if args.rows:
        wl = dataclasses.replace(wl, M=args.rows)
    return wl


def is_decode(wl):
    return wl.name.startswith("decode_")


def decode_copies(wl):
    """Distinct resident copies of a decode linear so that one step streams
    more than 4 x L2 of weights (packed codes + steps, 0.625 B per weight)."""
    lin = wl.linears[0]
    per = lin.N * lin.K * 5 // 8
    return max(1, -(-4 * L2_BYTES // per))


def decode_weight_passes(wl):
    """Weight passes of one open-mode decode step: the library runs the loops of
    a linear in one GEMV pass while their rows fit the GEMV's 16-row limit (at
    most 8 loops per launch)."""
    nbd = max(1, min(wl.T, 8, 16 // wl.M))
    return -(-wl.T // nbd)


def work_per_step(wl, copies=1):
    """Integer ops (2 per MAC) of one step and the rotation FLOPs (2 per FMA)."""
    ops = sum(2 * wl.M * lin.N * lin.K for lin in wl.linears) * wl.T * copies
    rot = sum(2 * wl.M * lin.K * (lin.a + lin.b) for lin in wl.linears) * wl.T * copies
    return ops, rot


def step_bytes(wl, copies=1):
    """Bytes one step reads from and writes to HBM at the least: the inputs,
    the resident weights (packed codes and steps) once per loop batch, the
    outputs."""
    x_el = 2 if wl.x_dtype == "bf16" else 4
    xb = sum(wl.M * lin.K * x_el for lin in wl.linears) * wl.T * copies
    yb = sum(wl.M * lin.N * 4 for lin in wl.linears) * wl.T * copies
    wb = sum(lin.N * lin.K * 5 // 8 for lin in wl.linears) * copies
    return xb, wb, yb


def workload_config(wl, world=1, copies=1):
    """The config dict both arms print (the same keys and values)."""
    x_el = 2 if wl.x_dtype == "bf16" else 4
    in_bytes = sum(wl.M * lin.K * x_el for lin in wl.linears) * wl.T * copies
    cfg = {"workload": wl.name, "M": wl.M, "T": wl.T, "a_bits": wl.a_bits, "group": 32,
           "linears": [[lin.name, lin.K, lin.N, lin.a, lin.b] for lin in wl.linears],
           "x_dtype": wl.x_dtype, "parallelism": f"replicas x{world}",
           "l2": ("inputs larger than L2 (%.1f GB per step), no flush" % (in_bytes / 1e9)
                  if in_bytes > 2 * L2_BYTES else
                  "flushed between timed steps (256 MiB write outside the events)")}
    if copies > 1:
        cfg["distinct_resident_copies"] = copies
    if wl.M != WORKLOADS[wl.name].M:
        cfg["rows_override"] = f"M = {wl.M} instead of {WORKLOADS[wl.name].M}"
    return cfg


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained") or d["bf16_tflops"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


def source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "bit_ptq_looped_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {"gemm": ["lq_gemm.cu", "lq_common.cuh"],
                  "rotate_quantize": ["lq_quant.cu", "lq_common.cuh"],
                  "gemv": ["lq_gemv.cu", "lq_common.cuh"]}


def ncu_traffic(kind, workload, units):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    is unchanged since the counters were taken; else None.  An entry taken on
    a smaller case of the same launch shape is scaled by the units processed
    (token rows per launch)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kind}/{workload}")
    if not e or e.get("source_hash") != source_hash(KERNEL_SOURCES[kind]):
        return None
    if e.get("rows_per_launch") and units:
        return e["bytes_per_launch"] * units / e["rows_per_launch"]
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_layers(wl):
    from oracle import lq_oracle as O

    return [O.OracleLayer(mp.W, mp.P1, mp.P2, mp.las, wl.a_bits)
            for mp in synth.module_params(wl)]


def oracle_sample(wl, rows, layers_o):
    """Run the oracle over `rows` token rows of every (loop, linear); returns seconds."""
    from oracle import lq_oracle as O

    xs = [[synth.loop_input(wl, lin, t, rows=np.arange(rows)) for lin in wl.linears]
          for t in range(wl.T)]
    t0 = time.perf_counter()
    for t in range(wl.T):
        for l, ol in enumerate(layers_o):
            O.loop_linear(xs[t][l], ol, t)
    return time.perf_counter() - t0


def cpu_oracle_rate(wl, target_s, layers_o):
    """Oracle throughput in TOPS on a bounded row sample sized for ~target_s seconds."""
    rows = min(wl.M, 8)
    dt = oracle_sample(wl, rows, layers_o)
    rows = int(min(wl.M, max(1, rows * target_s / max(dt, 1e-3) * 0.8)))
    dt = oracle_sample(wl, rows, layers_o)
    ops = sum(2 * rows * lin.N * lin.K for lin in wl.linears) * wl.T
    return dict(tops=ops / dt / 1e12, rows=rows, seconds=dt, tokens_per_s=rows / dt)


def cpu_baseline(wl, target_s):
    """The oracle as it stands on all host cores and on one core."""
    layers_o = oracle_layers(wl)
    r_all = cpu_oracle_rate(wl, target_s, layers_o)
    out = {"value": r_all["tops"], "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
           "tokens_per_s": r_all["tokens_per_s"],
           "sample": f"{r_all['rows']} of {wl.M} token rows through all {wl.T} loops x "
                     f"{len(wl.linears)} linears ({r_all['seconds']:.1f} s; rows are "
                     f"independent, so TOPS and tokens/s scale with rows)"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            r1 = cpu_oracle_rate(wl, target_s / 2, layers_o)
        out["one_core"] = {"value": r1["tops"], "unit": "TOPS", "cores": 1,
                           "tokens_per_s": r1["tokens_per_s"],
                           "sample": f"{r1['rows']} token rows ({r1['seconds']:.1f} s)"}
    except Exception as e:  # threadpoolctl missing: say so
        out["one_core"] = {"unavailable": str(e)}
    return out


def max_over_ranks(value_ms, world, device):
    """Max of a per-rank duration over all ranks (every rank takes part)."""
    if world <= 1:
        return float(value_ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, rank):
    if rank != 0:
        return
    wl = workload_of(args)
    layers_o = oracle_layers(wl)
    # every step is a bounded row sample sized so warm-up + steps take ~2 minutes
    per_step = min(5.0, max(0.01, 120.0 / max(1, args.steps + args.warmup)))
    r = cpu_oracle_rate(wl, per_step, layers_o)
    rows = r["rows"]
    for _ in range(args.warmup):
        oracle_sample(wl, rows, layers_o)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_sample(wl, rows, layers_o)
    ops = sum(2 * rows * lin.N * lin.K for lin in wl.linears) * wl.T * args.steps
    value = ops / total / 1e12
    cores = blas_threads()
    sample = (f"{rows} of {wl.M} token rows per step through all {wl.T} loops x "
              f"{len(wl.linears)} linears (rows are independent; TOPS scale with rows)")
    ms_sample = total / args.steps * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_sample,
        "ms_per_step_is": f"measured time of one sampled step ({rows} of {wl.M} rows)",
        "full_step_ms_extrapolated": ms_sample * wl.M / rows,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 quantizer, f64 rotation and GEMM",
        "data": "synthetic", "tokens_per_s": rows * args.steps / total,
        "config": workload_config(wl, 1),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
class Ctx:
    """Device, stream and timing helpers of one rank."""

    def __init__(self, torch, dist, dev, world):
        self.torch, self.dist, self.dev, self.world = torch, dist, dev, world
        self.stream = torch.cuda.current_stream(dev)
        self.flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)  # > 126 MB L2

    def barrier(self):
        self.torch.cuda.synchronize()
        if self.world > 1:
            self.dist.barrier()
        self.torch.cuda.synchronize()

    def timed(self, n, fn, flush_between=True):
        """Summed CUDA-event time (ms) of n calls of fn on the stream."""
        torch = self.torch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        self.barrier()
        for e0, e1 in evs:
            if flush_between:
                self.flush.zero_()
            e0.record(self.stream)
            fn()
            e1.record(self.stream)
        self.barrier()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs)


def build_layers(lq, torch, dev, wl, copies=1):
    """Fold with P^{-T} (host helper), pack, bind P and LAS; `copies` distinct
    resident copies of each linear (decode stacks)."""
    layers, packed = [], []
    for mp in synth.module_params(wl):
        Q1 = lq.lq_inverse_transpose(mp.P1).to(dev)
        Q2 = lq.lq_inverse_transpose(mp.P2).to(dev)
        Wf = lq.lq_fold_weights(torch.from_numpy(mp.W).to(dev), Q1, Q2)
        P1, P2 = torch.from_numpy(mp.P1).to(dev), torch.from_numpy(mp.P2).to(dev)
        for _ in range(copies):
            wq = lq.lq_pack_weights(Wf)
            packed.append(wq)
            layers.append(lq.lq_layer_create(wq, P1, P2, mp.las, wl.a_bits))
        del Wf
    return layers, packed


def free_layers(layers, packed):
    for l in layers:
        l.free()
    for w in packed:
        w.free()


def device_inputs(torch, dev, wl, copies=1):
    """The open-mode input buffer, (t, l) blocks of M x K back to back.  Up to
    8192 rows the seeded numpy recipe is used; larger workloads are drawn on
    the device with torch's generator (same recipe, another random stream)."""
    dt = torch.bfloat16 if wl.x_dtype == "bf16" else torch.float32
    n = wl.T * wl.M * sum(lin.K for lin in wl.linears) * copies
    x = torch.empty(n, dtype=dt, device=dev)
    off = 0
    for t in range(wl.T):
        for lin in wl.linears:
            if wl.M <= 8192:
                blk = torch.from_numpy(synth.loop_input(wl, lin, t).ravel()).to(dt).to(dev)
            else:
                blk = synth.device_loop_input(wl, lin, t, device=dev).reshape(-1)
            for _ in range(copies):
                x[off: off + blk.numel()] = blk
                off += blk.numel()
            del blk
    return x


def stack_fn(lq, layers, wl, x, y, ws, stream):
    def step():
        lq.lq_loop_stack(x, layers, wl.T, lq.LQ_OPEN, M=wl.M, y=y, ws=ws, stream=stream)
    return step


def probe_kernels(lq, ctx, step, n_probe, flush_between):
    """Per-kernel CUDA-event durations over a second timed region."""
    lq.lq_probe_enable(True)
    ctx.timed(n_probe, step, flush_between)
    pr = lq.lq_probe_read()
    lq.lq_probe_enable(False)
    kernels = {}
    for kind, (ms, cnt) in pr.items():
        if cnt:
            kernels[kind] = {"launches": cnt, "avg_us": ms / cnt * 1e3, "share": None}
    tot = sum(v["avg_us"] * v["launches"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["avg_us"] * v["launches"] / tot
    return kernels


def roofline_of(kernels, wl, n_probe, copies, peaks, sustained):
    """Roofline line of the dominant kernel: algorithmic work per launch over
    its average CUDA-event duration."""
    dom = max(kernels, key=lambda k: kernels[k]["avg_us"] * kernels[k]["launches"])
    avg_s = kernels[dom]["avg_us"] * 1e-6
    per_step = kernels[dom]["launches"] / n_probe  # launches of that kind per step
    T = wl.T
    bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    which = "sustained" if sustained else "burst"
    rows_per_launch = wl.M * T * copies / per_step * len(wl.linears)
    if dom == "gemm":
        flops = sum(2 * wl.M * lin.N * lin.K * T for lin in wl.linears) * copies / per_step
        r = {"bound": "tensor", "achieved": flops / avg_s / 1e12, "peak": 2.0 * bf16,
             "unit": "TFLOP/s",
             "peak_source": f"{peaks['source']} bf16 {which} x2 (8-bit/16-bit nominal ratio)"}
        # the unit that binds this kernel: the fp32 group rescale, 2 lane
        # operations (s_a*s_w, then the fused multiply-add) per output and group
        epi = sum(2 * wl.M * lin.N * (lin.K // 32) * T for lin in wl.linears) * copies / per_step
        epi_peak = SM_COUNT * FP32_LANES_PER_SM * SM_CLOCK_GHZ * 1e9 / 1e12
        r["epilogue_alu"] = {
            "achieved": epi / avg_s / 1e12, "peak": epi_peak, "unit": "T lane-ops/s",
            "frac": epi / avg_s / 1e12 / epi_peak,
            "peak_source": "derived: 148 SM x 128 FP32 lanes x 1.965 GHz"}
    elif dom == "rotate_quantize":
        flops = sum(2 * wl.M * lin.K * (lin.a + lin.b) * T for lin in wl.linears) * copies \
            / per_step
        peak = SM_COUNT * FP64_FMA_PER_SM_CLK * 2 * SM_CLOCK_GHZ * 1e9 / 1e12
        r = {"bound": "alu", "achieved": flops / avg_s / 1e12, "peak": peak,
             "unit": "TFLOP/s", "peak_source": "derived: 148 SM x 64 FP64 FMA/clk x 2 x 1.965 GHz"}
    else:  # GEMV: the weight streams (packed codes + steps) of a launch, each linear
        # once per weight pass, plus the float32 outputs; no L2 credit
        passes = decode_weight_passes(wl)
        wbytes = passes * sum(lin.N * lin.K * 5 // 8 for lin in wl.linears) * copies / per_step
        ybytes = sum(wl.M * lin.N * 4 * T for lin in wl.linears) * copies / per_step
        byts = wbytes + ybytes
        r = {"bound": "hbm", "achieved": byts / avg_s / 1e9, "peak": peaks["hbm_gbs"],
             "unit": "GB/s", "peak_source": peaks["source"] + " copy bandwidth",
             "bytes_per_launch": byts}
    r["frac"] = r["achieved"] / r["peak"]
    r["kernel"] = dom
    r["traffic"] = ncu_traffic(dom, wl.name, rows_per_launch)
    return r


def e2e_measure(lq, ctx, wl, layers, x_dev, y_dev, ws, n_steps):
    """The same step end to end through lq_loop_stack with host buffers: every
    step copies its inputs from pinned host memory and its outputs back.  The
    rows are processed in chunks on two device buffer sets (carved from the
    resident input and output buffers): the input copy of chunk i + 1 and the
    output copy of chunk i - 1 overlap chunk i's kernels.  The host input is
    the whole step's input (page-locked); the outputs land in a two-chunk
    page-locked host ring (a consumer drains it), because a whole step's
    output does not fit in the host's memory beside the input at the largest
    workload."""
    torch = ctx.torch
    T, M = wl.T, wl.M
    Ks = [lin.K for lin in wl.linears]
    Ns = [lin.N for lin in wl.linears]
    x_el = x_dev.element_size()
    row_in = T * sum(Ks)  # input elements per token row
    row_out = T * sum(Ns)
    Mc = M
    while Mc > 16384 and Mc % 2 == 0:
        Mc //= 2
    n_chunks = M // Mc
    # host input: the whole step, page-locked in place (exact size), unless the
    # ranks of this node would pin more than about 60 % of the free host memory;
    # then a two-chunk page-locked input ring whose chunks are sent again each
    # time (the same bytes cross the bus per step; the outputs are not checked)
    import psutil
    local = int(os.environ.get("LOCAL_WORLD_SIZE", ctx.world))
    nbytes = x_dev.numel() * x_el
    pinned = nbytes + 2 * Mc * row_out * 4
    in_ring = n_chunks > 2 and pinned * local > 0.6 * psutil.virtual_memory().available
    x_host = torch.empty(2 * Mc * row_in if in_ring else x_dev.numel(), dtype=x_dev.dtype)
    cudart = torch.cuda.cudart()
    assert int(cudart.cudaHostRegister(x_host.data_ptr(), x_host.numel() * x_el, 0)) == 0
    y_ring = torch.empty(2 * Mc * row_out, dtype=torch.float32)
    assert int(cudart.cudaHostRegister(y_ring.data_ptr(), y_ring.numel() * 4, 0)) == 0
    try:
        if in_ring:
            x_host.copy_(x_dev[:x_host.numel()])
        else:
            x_host.copy_(x_dev)
        slots = 1 if n_chunks == 1 else 2
        if n_chunks == 1:  # one chunk per step: separate device buffers, pipelined across steps
            xs = [x_dev, torch.empty_like(x_dev)]
            ys = [y_dev, torch.empty_like(y_dev)]
            slots = 2
        else:
            xs = [x_dev[i * Mc * row_in:(i + 1) * Mc * row_in] for i in range(2)]
            ys = [y_dev[i * Mc * row_out:(i + 1) * Mc * row_out] for i in range(2)]
        s_in, s_out = torch.cuda.Stream(ctx.dev), torch.cuda.Stream(ctx.dev)
        ev_in = [torch.cuda.Event() for _ in range(slots)]
        ev_comp = [torch.cuda.Event() for _ in range(slots)]
        ev_out = [torch.cuda.Event() for _ in range(slots)]
        stream = ctx.stream
        wl_c = dataclasses.replace(wl, M=Mc)

        def blocks(r0, rows, per_row, sizes):
            """(host/resident offset, chunk offset, length) of each (t, l) block."""
            out, off_full, off_c = [], 0, 0
            for t in range(T):
                for s in sizes:
                    out.append((off_full + r0 * s, off_c, rows * s))
                    off_full += M * s
                    off_c += rows * s
            return out

        in_blocks = [blocks(c * Mc, Mc, row_in, Ks) for c in range(n_chunks)]
        if in_ring:  # chunk c reads ring slot c % 2 (laid out as a chunk's blocks)
            in_blocks = [[((c % 2) * Mc * row_in + coff, coff, ln) for _, coff, ln in blk]
                         for c, blk in enumerate(in_blocks)]
        out_blocks = [blocks(0, Mc, row_out, Ns) for _ in range(1)][0]

        def run(n):
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            ctx.barrier()
            t0.record(stream)
            s_in.wait_event(t0)
            s_out.wait_event(t0)
            i = 0
            for _ in range(n):
                for c in range(n_chunks):
                    b = i % slots
                    if i >= slots:
                        s_in.wait_event(ev_comp[b])  # chunk i - slots has read xs[b]
                    with torch.cuda.stream(s_in):
                        for hoff, coff, ln in in_blocks[c]:
                            xs[b][coff:coff + ln].copy_(x_host[hoff:hoff + ln], non_blocking=True)
                    ev_in[b].record(s_in)
                    stream.wait_event(ev_in[b])
                    if i >= slots:
                        stream.wait_event(ev_out[b])  # chunk i - slots has left ys[b]
                    lq.lq_loop_stack(xs[b], layers, T, lq.LQ_OPEN, M=Mc, y=ys[b], ws=ws,
                                     stream=stream)
                    ev_comp[b].record(stream)
                    s_out.wait_event(ev_comp[b])
                    ring = y_ring[(b % 2) * Mc * row_out:(b % 2 + 1) * Mc * row_out]
                    with torch.cuda.stream(s_out):
                        for _, coff, ln in out_blocks:
                            ring[coff:coff + ln].copy_(ys[b][coff:coff + ln], non_blocking=True)
                    ev_out[b].record(s_out)
                    i += 1
            for b in range(slots):
                stream.wait_event(ev_out[b])
            t1.record(stream)
            ctx.barrier()
            return t0.elapsed_time(t1)

        run(1)  # records the chunk schedules
        ms = max_over_ranks(run(n_steps), ctx.world, ctx.dev)
    finally:
        torch.cuda.synchronize()
        cudart.cudaHostUnregister(x_host.data_ptr())
        cudart.cudaHostUnregister(y_ring.data_ptr())
    ops, _ = work_per_step(wl)
    return {"value": ops * n_steps * ctx.world / (ms * 1e-3) / 1e12, "unit": "TOPS",
            "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": M * row_out * 4,
            "ms_per_step": ms / n_steps, "steps": n_steps,
            "tokens_per_s": M * n_steps * ctx.world / (ms * 1e-3),
            "pipeline": f"{n_chunks} chunk(s) of {Mc} rows per step on two device buffer "
                        "sets; input copy of chunk i+1 and output copy of chunk i-1 overlap "
                        "chunk i's kernels",
            "host_buffers": ("two-chunk page-locked input ring (host memory would not hold "
                             "every rank's whole-step input)" if in_ring else
                             "whole-step input page-locked") +
                            "; outputs into a two-chunk page-locked host ring"}


def measure_stack(lq, ctx, wl, n_steps, warmup, n_probe, peaks, want_clocks=False):
    """Time the open-mode stack of a workload; returns its line (without e2e)."""
    torch = ctx.torch
    copies = decode_copies(wl) if is_decode(wl) else 1
    layers, packed = build_layers(lq, torch, ctx.dev, wl, copies)
    x = device_inputs(torch, ctx.dev, wl, copies)
    n_out = wl.T * wl.M * sum(lin.N for lin in wl.linears) * copies
    y = torch.empty(n_out, dtype=torch.float32, device=ctx.dev)
    # open mode with a workspace for all T loops: one quantize and one GEMM
    # launch per linear cover the T loops (the loops are independent here)
    ws = lq.workspace(layers, wl.M, ctx.dev, T=wl.T)
    big = x.numel() * x.element_size() > 2 * L2_BYTES
    step = stack_fn(lq, layers, wl, x, y, ws, ctx.stream)
    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    lq.lq_check_device(ctx.stream)
    sampler = ClockSampler(ctx.dev.index) if want_clocks else None
    if sampler:
        time.sleep(0.2)
    total_ms = ctx.timed(n_steps, step, flush_between=not big)
    clocks = sampler.stop() if sampler else None
    lq.lq_check_device(ctx.stream)
    total_ms = max_over_ranks(total_ms, ctx.world, ctx.dev)
    ops, rot = work_per_step(wl, copies)
    ms = total_ms / n_steps
    line = {"ms_per_step": ms, "TOPS": ops * ctx.world / (ms * 1e-3) / 1e12,
            "tokens_per_s": wl.M * copies * ctx.world / (ms * 1e-3),
            "rotation_tflops": rot * ctx.world / (ms * 1e-3) / 1e12,
            "clocks": clocks, "steps": n_steps, "config": workload_config(wl, ctx.world, copies)}
    kernels = probe_kernels(lq, ctx, step, n_probe, not big) if n_probe else None
    if is_decode(wl):
        xb, wb, yb = step_bytes(wl, copies)
        # weight passes per step: the loops batched into one GEMV pass share it
        passes = decode_weight_passes(wl)
        line["weight_passes_per_step"] = passes
        line["weight_bytes_per_step"] = passes * wb
        line["weight_stream_GB_s"] = passes * wb / (ms * 1e-3) / 1e9
        line["weight_stream_frac_hbm"] = line["weight_stream_GB_s"] / peaks["hbm_gbs"]
        line["tokens_per_s_per_linear"] = wl.M / (ms * 1e-3 / copies)
    if kernels:
        line["kernels"] = kernels
        line["launches_per_step"] = sum(v["launches"] for v in kernels.values()) / n_probe
        line["roofline"] = roofline_of(kernels, wl, n_probe, copies, peaks,
                                       sustained=total_ms > 1000.0)
    return line, (layers, packed, x, y, ws, copies)


def aux_schedules(lq, ctx, wl, layers, x_dev, ops_step):
    """The same step under other schedules of the loop driver: loop by loop
    (workspace for one loop), and SLT serving with every module selected (its
    own transform and weight at every loop, so no loop shares a launch)."""
    torch, dev, stream, timed = ctx.torch, ctx.dev, ctx.stream, ctx.timed
    params = synth.module_params(wl)
    out = {}
    M, T, L = wl.M, wl.T, len(wl.linears)
    y = torch.empty(T * M * sum(lin.N for lin in wl.linears), dtype=torch.float32, device=dev)
    n = 50

    ws1 = lq.workspace(layers, M, dev)
    run = lambda: lq.lq_loop_stack(x_dev, layers, T, lq.LQ_OPEN, M=M, y=y, ws=ws1,
                                   stream=stream)
    for _ in range(3):
        run()
    ms = timed(n, run) / n
    out["loop_by_loop"] = {"ms_per_step": ms, "TOPS": ops_step / (ms * 1e-3) / 1e12,
                           "launches_per_step": 2 * T * L}

    lins = wl.linears
    if all(lins[l].N == lins[(l + 1) % L].K for l in range(L)):
        # chain mode: loops strictly in sequence, y of each step feeding the next
        # (inputs: the first step's x), plain and with CTA at the T - 1 transitions
        x0 = x_dev[: M * lins[0].K]
        run = lambda: lq.lq_loop_stack(x0, layers, T, lq.LQ_CHAIN, M=M, y=y, ws=ws1,
                                       stream=stream)
        for _ in range(3):
            run()
        ms = timed(n, run) / n
        out["chain"] = {"ms_per_step": ms, "TOPS": ops_step / (ms * 1e-3) / 1e12}
        d = lins[-1].N
        rng = np.random.default_rng(23)
        U = torch.from_numpy((0.05 * rng.standard_normal((d, 8))).astype(np.float32)).to(dev)
        V = torch.from_numpy((0.05 * rng.standard_normal((d, 8))).astype(np.float32)).to(dev)
        a = torch.from_numpy((1 + 0.1 * rng.standard_normal((T - 1, d))).astype(np.float32)).to(dev)
        b = torch.from_numpy((0.1 * rng.standard_normal((T - 1, d))).astype(np.float32)).to(dev)
        cta = lq.lq_cta_create(U, V, a, b, rng.uniform(0.1, 0.9, T - 1))
        ws_c = torch.empty(lq.lq_cta_stack_workspace_bytes(layers, M), dtype=torch.uint8,
                           device=dev)
        run = lambda: lq.lq_loop_stack_cta(x0, layers, T, cta, M=M, y=y, ws=ws_c, stream=stream)
        for _ in range(3):
            run()
        ms_c = timed(n, run) / n
        out["chain_cta"] = {"ms_per_step": ms_c, "TOPS": ops_step / (ms_c * 1e-3) / 1e12,
                            "transitions": T - 1,
                            "us_per_transition": (ms_c - ms) * 1e3 / max(T - 1, 1)}
        cta.free()

    # trajectory Hessian of the first module over its T loop inputs (bf16)
    lin0 = lins[0]
    if wl.x_dtype == "bf16" and lin0.K % 128 == 0:
        K0 = lin0.K
        xh = torch.empty(T * M * K0, dtype=torch.bfloat16, device=dev)
        off = 0
        for t in range(T):  # loop t's input of module 0 inside the open-mode buffer
            src = x_dev[(t * sum(l.K for l in lins)) * M: (t * sum(l.K for l in lins) + K0) * M]
            xh[off: off + M * K0] = src
            off += M * K0
        Hh = torch.empty((K0, K0), dtype=torch.float32, device=dev)
        wsh = torch.empty(lq.lib().lq_hessian_workspace_bytes(M, K0, T), dtype=torch.uint8,
                          device=dev)
        run = lambda: lq.lq_trajectory_hessian(xh, T, M=M, H=Hh, ws=wsh, stream=stream)
        for _ in range(3):
            run()
        ms_h = timed(n, run) / n
        flops = T * M * K0 * (K0 + 1)  # the symmetric product: one multiply-add per pair i <= j
        peaks = load_peaks()
        out["trajectory_hessian"] = {
            "workload": f"H = sum_t X_t^T X_t, T={T} x {M} x {K0} bf16 -> {K0}x{K0} fp32",
            "us": ms_h * 1e3, "TFLOP_s": flops / (ms_h * 1e-3) / 1e12,
            "frac_bf16_peak": flops / (ms_h * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "flops": flops, "includes": "bf16 transpose of the inputs (one launch) + the product"}
        del xh, Hh, wsh

    rng = np.random.default_rng(17)
    own, keep = [], []
    for t in range(T):
        row = []
        for mp in params:
            a, b = mp.P1.shape[0], mp.P2.shape[0]
            P1 = np.linalg.qr(rng.standard_normal((a, a)))[0].astype(np.float32)
            P2 = np.linalg.qr(rng.standard_normal((b, b)))[0].astype(np.float32)
            Q1 = lq.lq_inverse_transpose(P1).to(dev)
            Q2 = lq.lq_inverse_transpose(P2).to(dev)
            Wf = lq.lq_fold_weights(torch.from_numpy(mp.W).to(dev), Q1, Q2)
            wq = lq.lq_pack_weights(Wf)
            del Wf
            row.append(lq.lq_layer_create(wq, torch.from_numpy(P1).to(dev),
                                          torch.from_numpy(P2).to(dev), mp.las, wl.a_bits))
            keep.append(wq)
        own.append(row)
    ws2 = lq.workspace(layers, M, dev, T=T)
    run = lambda: lq.lq_loop_stack_slt(x_dev, own, lq.LQ_OPEN, M=M, y=y, ws=ws2, stream=stream)
    for _ in range(3):
        run()
    ms = timed(n, run) / n
    shared_bytes = sum(l.wq.info()["device_bytes"] for l in layers)
    out["slt_all_selected"] = {"ms_per_step": ms, "TOPS": ops_step / (ms * 1e-3) / 1e12,
                               "resident_weight_bytes": T * shared_bytes,
                               "shared_weight_bytes": shared_bytes}
    for row in own:
        for l in row:
            l.free()
    for wq in keep:
        wq.free()
    return out


def aux_decode_chain(lq, ctx, peaks, M=4, L=32):
    """Decode as a real looped model runs it: chain mode, each (t, l) step's
    input the previous step's output, so the T x L quantize -> GEMV pairs are
    strictly sequential (K = N = 2048, L distinct resident copies, W4A8)."""
    torch = ctx.torch
    wl = synth.decode_workload(M, 2048, 8)
    layers, packed = build_layers(lq, torch, ctx.dev, wl, L)
    x0 = torch.from_numpy(synth.loop_input(wl, wl.linears[0], 0)).to(torch.bfloat16).to(ctx.dev)
    y = torch.empty(wl.T * L * M * 2048, dtype=torch.float32, device=ctx.dev)
    ws = lq.workspace(layers, M, ctx.dev)

    def step():
        lq.lq_loop_stack(x0, layers, wl.T, lq.LQ_CHAIN, M=M, y=y, ws=ws, stream=ctx.stream)

    for _ in range(3):
        step()
    n = 20
    ms = ctx.timed(n, step) / n
    free_layers(layers, packed)
    wb = 2048 * 2048 * 5 // 8
    return {"workload": f"W4A8 M={M} K=N=2048, chain mode, T={wl.T} x {L} distinct linears",
            "ms_per_step": ms, "us_per_linear": ms * 1e3 / (wl.T * L),
            "tokens_per_s": M / (ms * 1e-3),
            "weight_stream_frac_hbm": wl.T * L * wb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}


def aux_hbm_kernels(lq, ctx, peaks):
    """The quantize-only kernel and the streaming GEMV on launches far larger than L2."""
    torch, dev, stream = ctx.torch, ctx.dev, ctx.stream
    out = {}
    M, K = 65536, 2048
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    xt = torch.randn((M, K), generator=g, device=dev, dtype=torch.float32)
    codes = torch.empty((M, K), dtype=torch.int8, device=dev)
    sc = torch.empty((M, K // 32), dtype=torch.float32, device=dev)

    def q_step():
        lq.lq_quantize_act(xt, None, None, 0.85, 4, codes8=codes, scales=sc, stream=stream)

    for _ in range(3):
        q_step()
    ms = ctx.timed(20, q_step, flush_between=False) / 20
    byts = M * K * 4 + M * K + M * (K // 32) * 4
    out["quantize_only"] = {"workload": f"{M}x{K} fp32 -> int8 codes + fp32 steps",
                            "us": ms * 1e3, "GB_s": byts / (ms * 1e-3) / 1e9,
                            "frac_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                            "bytes_per_launch": byts}
    del xt, codes, sc
    # the GEMV kernel's streaming rate on one large launch: W4A8, M = 1, 4, 16,
    # K = 2048, N = 36 x 5632 weight rows (263 MB packed, > 2x L2)
    wl = synth.decode_workload(4, 5632, 8)
    (mp,) = synth.module_params(wl)
    Q1 = lq.lq_inverse_transpose(mp.P1).to(dev)
    Q2 = lq.lq_inverse_transpose(mp.P2).to(dev)
    P1, P2 = torch.from_numpy(mp.P1).to(dev), torch.from_numpy(mp.P2).to(dev)
    Nb = 36 * 5632
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    Wb = torch.randn((Nb, 2048), generator=g, device=dev, dtype=torch.float32) * 0.02
    Wf = lq.lq_fold_weights(Wb, Q1, Q2)
    del Wb
    wqb = lq.lq_pack_weights(Wf)
    del Wf
    lb = lq.lq_layer_create(wqb, P1, P2, mp.las, 8)
    for Ms in (1, 4, 16):
        xb = torch.from_numpy(synth.loop_input(synth.decode_workload(Ms, 5632, 8),
                                               wl.linears[0], 0)).to(torch.bfloat16).to(dev)
        yb = torch.empty((Ms, Nb), dtype=torch.float32, device=dev)
        wsb = lq.workspace([lb], Ms, dev)

        def b_step():
            lq.lq_loop_linear(xb, lb, 0, y=yb, ws=wsb, stream=stream)

        for _ in range(3):
            b_step()
        lq.lq_probe_enable(True)
        ctx.timed(10, b_step, flush_between=False)
        pr = lq.lq_probe_read()
        lq.lq_probe_enable(False)
        gemv_ms, gemv_n = pr["gemv"]
        avg = gemv_ms / max(gemv_n, 1)
        byts = Nb * 2048 // 2 + Nb * 64 * 4 + Ms * 2048 + Ms * 64 * 8 + Ms * Nb * 4
        out[f"gemv_stream_M{Ms}"] = {
            "workload": f"W4A8 M={Ms} K=2048 N={Nb}, one launch", "us": avg * 1e3,
            "bytes_per_launch": byts, "GB_s": byts / (avg * 1e-3) / 1e9,
            "frac_hbm": byts / (avg * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    lb.free()
    wqb.free()
    return out


def run_lq(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bit_ptq_looped_b200 import build as B
    from bit_ptq_looped_b200 import lq

    if rank == 0:
        B.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ctx = Ctx(torch, dist, dev, world)
    peaks = load_peaks()
    wl = workload_of(args)

    n_probe = 0 if args.no_probe else min(args.steps, 5 if wl.M > 65536 else 200)
    line, held = measure_stack(lq, ctx, wl, args.steps, args.warmup, n_probe, peaks,
                               want_clocks=True)
    layers, packed, x, y, ws, copies = held
    e2e = None
    if not args.no_e2e:
        n_e2e = 2 if wl.M > 65536 else min(args.steps, 50)
        e2e = e2e_measure(lq, ctx, wl, layers, x, y, ws, n_e2e)
    free_layers(layers, packed)
    del x, y, ws, held
    torch.cuda.empty_cache()

    aux = None
    if not args.no_aux:
        aux = {}
        for name in AUX_WORKLOADS:
            if name == wl.name:
                continue
            awl = WORKLOADS[name]
            steps = 10 if is_decode(awl) else 100
            a_line, a_held = measure_stack(lq, ctx, awl, steps, 3, steps, peaks)
            if name == synth.ATTN_PROJ.name:
                # the same linear under the driver's other schedules (loop by
                # loop, chain, chain with loop-transition adapters, SLT serving)
                # and the trajectory Hessian of its loop inputs
                a_line["schedules"] = aux_schedules(lq, ctx, awl, a_held[0], a_held[2],
                                                    work_per_step(awl)[0])
            free_layers(a_held[0], a_held[1])
            del a_held
            aux[name] = a_line
        torch.cuda.empty_cache()
        aux["decode_chain_M4_N2048"] = aux_decode_chain(lq, ctx, peaks)
        aux.update(aux_hbm_kernels(lq, ctx, peaks))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    if rank == 0:
        launches = line.get("launches_per_step")
        out = {
            "metric": METRIC, "value": line["TOPS"], "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": line["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "int4 codes (int32/fp32 group sums), fp32 rescale, fp64 rotation",
            "data": "synthetic", "tokens_per_s": line["tokens_per_s"],
            "rotation_tflops": line["rotation_tflops"],
            "config": line["config"],
            "roofline": line.get("roofline"), "kernels": line.get("kernels"),
            "aux": aux, "cpu_baseline": cpu, "e2e": e2e, "clocks": line["clocks"],
            "gpu_launches": None if launches is None else int(round(launches * args.steps)),
        }
        if is_decode(wl):
            out["decode"] = {k: line[k] for k in (
                "weight_passes_per_step", "weight_bytes_per_step", "weight_stream_GB_s",
                "weight_stream_frac_hbm", "tokens_per_s_per_linear") if k in line}
        print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    distributed = world > 1 and args.impl == "lq"
    if distributed:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group(backend="nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank)
        else:
            run_lq(args, rank, world, local_rank)
    finally:
        if distributed:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
