#!/usr/bin/env python
"""Benchmark of the W4A4 looped quantized linear on B200 (one JSON line).

A step is one pass of the whole hot path over one batch: for each of the T
loops, the fused Kronecker-rotate + group-32 LAS quantizer and the
group-rescaled integer GEMM of every shared linear of the workload
(lq_loop_stack, open mode, weights resident).  Default workload: the
Ouro-1.4B-shaped attention projection K = N = 2048, M = 2048 tokens, T = 4.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lq|reference]

With torchrun (N > 1) every rank runs its own replica of the workload on its
GPU (no data-path collective; weak scaling); the time is the max over ranks.
`--impl reference` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
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

WORKLOADS = {w.name: w for w in (synth.TINY, synth.ATTN_PROJ, synth.MLP)}
DEFAULT_WORKLOAD = synth.ATTN_PROJ.name
METRIC = "W4A4 looped-linear TOPS & tokens/s at 1 B200; % of int8 tensor/HBM roofline"
SM_COUNT = 148
SM_CLOCK_GHZ = 1.965
FP64_FMA_PER_SM_CLK = 64  # B200 FP64 units per SM
FP32_LANES_PER_SM = 128  # FP32 FMA lanes per SM


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["lq", "reference"], default="lq")
    p.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-probe", action="store_true")
    p.add_argument("--no-aux", action="store_true",
                   help="skip the quantize-only and decode-GEMV bandwidth measurements")
    return p.parse_args()


def work_per_step(wl):
    """Integer ops (2 per MAC) of one step and the rotation FLOPs (2 per FMA)."""
    ops = sum(2 * wl.M * lin.N * lin.K for lin in wl.linears) * wl.T
    rot = sum(2 * wl.M * lin.K * (lin.a + lin.b) for lin in wl.linears) * wl.T
    return ops, rot


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
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


def ncu_traffic(kind, workload):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    is unchanged since the counters were taken; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kind}/{workload}")
    if not e or e.get("source_hash") != source_hash(KERNEL_SOURCES[kind]):
        return None
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


def cpu_oracle_rate(wl, target_s):
    """Oracle throughput in TOPS on a bounded row sample sized for ~target_s seconds."""
    from oracle import lq_oracle as O

    layers_o = [O.OracleLayer(mp.W, mp.P1, mp.P2, mp.las, wl.a_bits)
                for mp in synth.module_params(wl)]
    rows = 8
    dt = oracle_sample(wl, rows, layers_o)
    rows = int(min(wl.M, max(1, rows * target_s / max(dt, 1e-3) * 0.8)))
    dt = oracle_sample(wl, rows, layers_o)
    ops = sum(2 * rows * lin.N * lin.K for lin in wl.linears) * wl.T
    return dict(tops=ops / dt / 1e12, rows=rows, seconds=dt, layers=layers_o,
                tokens_per_s=rows / dt)


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
    wl = WORKLOADS[args.workload]
    ops_step, _ = work_per_step(wl)
    # every step is a bounded row sample sized so warm-up + steps take ~2 minutes
    per_step = min(5.0, max(0.01, 120.0 / max(1, args.steps + args.warmup)))
    r = cpu_oracle_rate(wl, per_step)
    rows = r["rows"]
    for _ in range(args.warmup):
        oracle_sample(wl, rows, r["layers"])
    total = 0.0
    for _ in range(args.steps):
        total += oracle_sample(wl, rows, r["layers"])
    ops = sum(2 * rows * lin.N * lin.K for lin in wl.linears) * wl.T * args.steps
    value = ops / total / 1e12
    cores = blas_threads()
    sample = (f"{rows} of {wl.M} token rows per step through all {wl.T} loops x "
              f"{len(wl.linears)} linears (rows are independent; TOPS scale with rows)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3 * wl.M / rows, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 quantizer, f64 rotation and GEMM",
        "data": "synthetic", "tokens_per_s": rows * args.steps / total,
        "config": {"workload": wl.name, "M": wl.M, "T": wl.T, "a_bits": wl.a_bits, "group": 32,
                   "linears": [[lin.name, lin.K, lin.N] for lin in wl.linears]},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# HBM-bound kernels of the path, measured on inputs far larger than L2
# ---------------------------------------------------------------------------
def aux_hbm_kernels(lq, torch, dev, stream, timed, peaks):
    out = {}
    # quantize-only (already transformed fp32 input): 65536 x 2048 fp32 = 512 MiB read
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
    n = 20
    ms = timed(n, q_step, flush_between=False) / n
    byts = M * K * 4 + M * K + M * (K // 32) * 4
    out["quantize_only"] = {"workload": f"{M}x{K} fp32 -> int8 codes + fp32 steps",
                            "us": ms * 1e3, "GB_s": byts / (ms * 1e-3) / 1e9,
                            "frac_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                            "bytes_per_launch": byts}
    del xt, codes, sc
    # decode GEMV: W4A8, M = 4 tokens, K = 2048, N = 5632, T = 4 loops over a
    # stack of 72 distinct resident linears (7.2 MB of packed weights + steps
    # each, 519 MB in all, > 4x L2), one weight stream per loop and linear
    wl = synth.decode_workload(4, 5632, 8)
    (mp,) = synth.module_params(wl)
    Q1 = lq.lq_inverse_transpose(mp.P1).to(dev)
    Q2 = lq.lq_inverse_transpose(mp.P2).to(dev)
    Wf = lq.lq_fold_weights(torch.from_numpy(mp.W).to(dev), Q1, Q2)
    P1, P2 = torch.from_numpy(mp.P1).to(dev), torch.from_numpy(mp.P2).to(dev)
    L = 72
    wqs = [lq.lq_pack_weights(Wf) for _ in range(L)]
    layers = [lq.lq_layer_create(w, P1, P2, mp.las, 8) for w in wqs]
    del Wf
    Md, T = wl.M, wl.T
    x = torch.from_numpy(np.concatenate([synth.loop_input(wl, wl.linears[0], t).ravel()
                                         for t in range(T) for _ in range(L)]))
    x = x.to(torch.bfloat16).to(dev)
    y = torch.empty(T * L * Md * 5632, dtype=torch.float32, device=dev)
    ws = lq.workspace(layers, Md, dev)

    def d_step():
        lq.lq_loop_stack(x, layers, T, lq.LQ_OPEN, M=Md, y=y, ws=ws, stream=stream)

    for _ in range(3):
        d_step()
    n = 10
    step_ms = timed(n, d_step, flush_between=False) / n
    lq.lq_probe_enable(True)
    timed(n, d_step, flush_between=False)
    pr = lq.lq_probe_read()
    lq.lq_probe_enable(False)
    gemv_ms, gemv_n = pr["gemv"]
    per_launch = 5632 * 2048 // 2 + 5632 * 64 * 4 + Md * 2048 + Md * 64 * 8 + Md * 5632 * 4
    avg = gemv_ms / max(gemv_n, 1)
    out["gemv_decode"] = {
        "workload": f"W4A8 M={Md} K=2048 N=5632, T={T} x {L} distinct linears",
        "gemv_us": avg * 1e3, "GB_s": per_launch / (avg * 1e-3) / 1e9,
        "frac_hbm": per_launch / (avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "bytes_per_launch": per_launch,
        "step_ms": step_ms, "tokens_per_s": Md / (step_ms * 1e-3),
        # the whole stack as one weight stream: T x L launches' bytes over the step
        "stream_GB_s": T * L * per_launch / (step_ms * 1e-3) / 1e9,
        "stream_frac_hbm": T * L * per_launch / (step_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "rotate_quantize_us": pr["rotate_quantize"][0] / max(pr["rotate_quantize"][1], 1) * 1e3}
    for l in layers:
        l.free()
    for w in wqs:
        w.free()
    del x, y, ws
    # the GEMV kernel's streaming rate on one large launch: W4A8, M = 1, 4, 16, K = 2048,
    # N = 36 x 5632 weight rows (263 MB packed, > 2x L2), seeded N(0, 0.02) weights
    Nb = 36 * 5632
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    Wb = torch.randn((Nb, 2048), generator=g, device=dev, dtype=torch.float32) * 0.02
    Wf = lq.lq_fold_weights(Wb, Q1, Q2)
    del Wb
    wqb = lq.lq_pack_weights(Wf)
    del Wf
    lb = lq.lq_layer_create(wqb, P1, P2, mp.las, 8)
    for Ms in (1, 4, 16):  # decode row counts of the decode configuration
        xb = torch.from_numpy(synth.loop_input(synth.decode_workload(Ms, 5632, 8),
                                               wl.linears[0], 0)).to(torch.bfloat16).to(dev)
        yb = torch.empty((Ms, Nb), dtype=torch.float32, device=dev)
        wsb = lq.workspace([lb], Ms, dev)

        def b_step():
            lq.lq_loop_linear(xb, lb, 0, y=yb, ws=wsb, stream=stream)

        for _ in range(3):
            b_step()
        lq.lq_probe_enable(True)
        timed(10, b_step, flush_between=False)
        pr = lq.lq_probe_read()
        lq.lq_probe_enable(False)
        gemv_ms, gemv_n = pr["gemv"]
        avg = gemv_ms / max(gemv_n, 1)
        byts = Nb * 2048 // 2 + Nb * 64 * 4 + Ms * 2048 + Ms * 64 * 8 + Ms * Nb * 4
        out["gemv_stream" if Ms == 4 else f"gemv_stream_M{Ms}"] = {
            "workload": f"W4A8 M={Ms} K=2048 N={Nb}, one launch", "us": avg * 1e3,
            "bytes_per_launch": byts, "GB_s": byts / (avg * 1e-3) / 1e9,
            "frac_hbm": byts / (avg * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    lb.free()
    wqb.free()
    return out


def aux_schedules(lq, torch, dev, stream, timed, wl, params, layers, x_dev, ops_step):
    """The same step under other schedules of the loop driver: loop by loop
    (workspace for one loop), and SLT serving with every module selected (its
    own transform and weight at every loop, so no loop shares a launch)."""
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


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
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
    wl = WORKLOADS[args.workload]
    params = synth.module_params(wl)

    # resident layers: fold with P^{-T} (host helper), pack, bind P and LAS
    layers, keep = [], []
    for mp in params:
        Q1 = lq.lq_inverse_transpose(mp.P1).to(dev)
        Q2 = lq.lq_inverse_transpose(mp.P2).to(dev)
        Wf = lq.lq_fold_weights(torch.from_numpy(mp.W).to(dev), Q1, Q2)
        wq = lq.lq_pack_weights(Wf)
        P1, P2 = torch.from_numpy(mp.P1).to(dev), torch.from_numpy(mp.P2).to(dev)
        layers.append(lq.lq_layer_create(wq, P1, P2, mp.las, wl.a_bits))
        keep.append((wq, Wf))
        del Wf
    M, T, L = wl.M, wl.T, len(wl.linears)
    xs = [synth.loop_input(wl, lin, t) for t in range(T) for lin in wl.linears]
    x_host = torch.from_numpy(np.concatenate([x.ravel() for x in xs]))
    x_host = (x_host.to(torch.bfloat16) if wl.x_dtype == "bf16" else x_host).pin_memory()
    x_dev = x_host.to(dev)
    n_out = T * M * sum(lin.N for lin in wl.linears)
    y = torch.empty(n_out, dtype=torch.float32, device=dev)
    y_host = torch.empty(n_out, dtype=torch.float32).pin_memory()
    # open mode with a workspace for all T loops: one quantize and one GEMM
    # launch per linear cover the T loops (the loops are independent here)
    ws = lq.workspace(layers, M, dev, T=T)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def step():
        lq.lq_loop_stack(x_dev, layers, T, lq.LQ_OPEN, M=M, y=y, ws=ws, stream=stream)

    def timed(n, fn, flush_between=True):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            if flush_between:
                flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in evs)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    lq.lq_check_device(stream)

    sampler = ClockSampler(local_rank)
    time.sleep(0.2)
    total_ms = timed(args.steps, step)
    clocks = sampler.stop()
    lq.lq_check_device(stream)
    total_ms = max_over_ranks(total_ms, world, dev)

    ops_step, rot_step = work_per_step(wl)
    loops_per_launch = min(T, 8) if M > 16 else 1  # the driver's open-mode batching
    value = ops_step * args.steps * world / (total_ms * 1e-3) / 1e12
    ms_per_step = total_ms / args.steps
    tokens_per_s = M * args.steps * world / (total_ms * 1e-3)

    # kernel probe: per-kernel CUDA-event durations over a second timed region
    kernels, roofline = {}, None
    if not args.no_probe:
        n_probe = min(args.steps, 200)
        lq.lq_probe_enable(True)
        timed(n_probe, step)
        pr = lq.lq_probe_read()
        lq.lq_probe_enable(False)
        peaks = load_peaks()
        for kind, (ms, cnt) in pr.items():
            if cnt:
                kernels[kind] = {"launches": cnt, "avg_us": ms / cnt * 1e3,
                                 "share": None}
        tot = sum(v["avg_us"] * v["launches"] for v in kernels.values())
        for v in kernels.values():
            v["share"] = v["avg_us"] * v["launches"] / tot
        dom = max(kernels, key=lambda k: kernels[k]["avg_us"] * kernels[k]["launches"])
        avg_s = kernels[dom]["avg_us"] * 1e-6
        per_step = kernels[dom]["launches"] / n_probe  # launches of that kind per step
        if dom == "gemm":
            flops = sum(2 * M * lin.N * lin.K * T for lin in wl.linears) / per_step
            peak = 2.0 * peaks["bf16_tflops"]  # 8-bit dense = 2x bf16 dense (nominal ratio)
            roofline = {"bound": "tensor", "achieved": flops / avg_s / 1e12, "peak": peak,
                        "unit": "TFLOP/s", "peak_source": peaks["source"] +
                        " bf16 burst x2 (8-bit/16-bit nominal ratio)"}
            # the unit that binds this kernel: the fp32 group rescale, 2 lane
            # operations (s_a*s_w, then the fused multiply-add) per output and group
            epi = sum(2 * M * lin.N * (lin.K // 32) * T for lin in wl.linears) / per_step
            epi_peak = SM_COUNT * FP32_LANES_PER_SM * SM_CLOCK_GHZ * 1e9 / 1e12
            roofline["epilogue_alu"] = {
                "achieved": epi / avg_s / 1e12, "peak": epi_peak, "unit": "T lane-ops/s",
                "frac": epi / avg_s / 1e12 / epi_peak,
                "peak_source": "derived: 148 SM x 128 FP32 lanes x 1.965 GHz"}
        elif dom == "rotate_quantize":
            flops = sum(2 * M * lin.K * (lin.a + lin.b) * T for lin in wl.linears) / per_step
            peak = SM_COUNT * FP64_FMA_PER_SM_CLK * 2 * SM_CLOCK_GHZ * 1e9 / 1e12
            roofline = {"bound": "alu", "achieved": flops / avg_s / 1e12, "peak": peak,
                        "unit": "TFLOP/s", "peak_source":
                        "derived: 148 SM x 64 FP64 FMA/clk x 2 x 1.965 GHz"}
        else:
            byts = sum((lin.N * lin.K // 2 + lin.N * lin.K // 8) * T
                       for lin in wl.linears) / per_step
            roofline = {"bound": "hbm", "achieved": byts / avg_s / 1e9, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "peak_source": peaks["source"]}
        roofline["frac"] = roofline["achieved"] / roofline["peak"]
        roofline["kernel"] = dom
        roofline["traffic"] = ncu_traffic(dom, wl.name)

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        n_e2e = min(args.steps, 50)

        def e2e_step():
            x_dev.copy_(x_host, non_blocking=True)
            step()
            y_host.copy_(y, non_blocking=True)

        serial_ms = max_over_ranks(timed(n_e2e, e2e_step), world, dev)
        # the same steps pipelined: two device buffer sets, the input copy of
        # step i + 1 and the output copy of step i - 1 on their own streams,
        # overlapping step i's kernels (PCIe copies in both directions at once)
        xs = [x_dev, torch.empty_like(x_dev)]
        ys = [y, torch.empty_like(y)]
        yh = [y_host, torch.empty_like(y_host).pin_memory()]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def pipelined(n):
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            t0.record(stream)
            s_in.wait_event(t0)
            for i in range(n):
                b = i % 2
                if i >= 2:
                    s_in.wait_event(ev_comp[b])  # step i - 2 has read xs[b]
                with torch.cuda.stream(s_in):
                    xs[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])  # step i - 2's output has left ys[b]
                lq.lq_loop_stack(xs[b], layers, T, lq.LQ_OPEN, M=M, y=ys[b], ws=ws,
                                 stream=stream)
                ev_comp[b].record(stream)
                s_out.wait_event(ev_comp[b])
                with torch.cuda.stream(s_out):
                    yh[b].copy_(ys[b], non_blocking=True)
                ev_out[b].record(s_out)
            stream.wait_event(ev_out[(n - 1) % 2])
            stream.wait_event(ev_out[n % 2])
            t1.record(stream)
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            return t0.elapsed_time(t1)

        pipelined(4)  # record the schedule for the second buffer set
        e2e_ms = max_over_ranks(pipelined(n_e2e), world, dev)
        e2e = {"value": ops_step * n_e2e * world / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS",
               "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
               "d2h_bytes_per_step": y_host.numel() * y_host.element_size(),
               "ms_per_step": e2e_ms / n_e2e,
               "pipelined": "copy-in of step i+1 and copy-out of step i-1 overlap step i",
               "serial_value": ops_step * n_e2e * world / (serial_ms * 1e-3) / 1e12}

    aux = None
    if not args.no_aux:
        aux = aux_hbm_kernels(lq, torch, dev, stream, timed, load_peaks())
        aux.update(aux_schedules(lq, torch, dev, stream, timed, wl, params, layers, x_dev,
                                 ops_step))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = cpu_oracle_rate(wl, args.cpu_seconds)
        cpu = {"value": r["tops"], "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{r['rows']} of {M} token rows through all {T} loops x {L} linears "
                         f"({r['seconds']:.1f} s; rows are independent)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4 codes (int32/fp32 group sums), fp32 rescale, fp64 rotation",
            "data": "synthetic", "tokens_per_s": tokens_per_s,
            "rotation_tflops": rot_step * args.steps * world / (total_ms * 1e-3) / 1e12,
            "config": {"workload": wl.name, "M": M, "T": T, "a_bits": wl.a_bits, "group": 32,
                       "linears": [[lin.name, lin.K, lin.N, lin.a, lin.b] for lin in wl.linears],
                       "x_dtype": wl.x_dtype, "parallelism": f"replicas x{world}",
                       "loops_per_launch": loops_per_launch,
                       "l2": "flushed between timed steps (256 MiB write outside the events)"},
            "roofline": roofline, "kernels": kernels, "aux": aux, "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks, "gpu_launches": 2 * L * -(-T // loops_per_launch) * args.steps,
        }
        print(json.dumps(line), flush=True)
    for l in layers:
        l.free()
    for wq, _ in keep:
        wq.free()


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
