"""Seeded synthetic inputs for the looped quantized linear.

This module only draws numbers: activations with fixed outlier channels and a
per-loop drift, Gaussian weights, random orthogonal Kronecker factors and
per-loop LAS clip scalars.  It holds none of the method's arithmetic (no
rotation, no quantization, no GEMM), so both the CUDA path and the CPU oracle
can be fed from it.

Shapes follow an Ouro-1.4B-sized looped transformer: 24 layers run 4 times per
token, hidden size 2048, MLP width 5632, calibration samples of 256 tokens
(LoopQ reproduction README, "LoopQ 4-bit quantization of Ouro-1.4B" header;
paper_specification.yaml, experiment_hyperparameters; the Ouro down_proj input
dimension 5632 from "Quantizing Looped Transformers", Table 19).  The pages
measure on Pile text and lm-eval tasks; these draws stand in for them.

Recipe (every number is float32 unless noted):
  * base activation x ~ N(0, 1) drawn in float64 and rounded to float32;
  * outlier channels: ``round(frac * K)`` distinct channels chosen once per
    module, multiplied by ``mult`` for every token and loop;
  * loop drift: x_t = fl32(fl32((1 + 0.25 t) * x) + fl32(0.1 t)), t = 0..T-1;
  * bf16 workloads round x_t to bfloat16 (round-to-nearest-even);
  * W ~ N(0, 0.02) (float32);
  * P1, P2 = Q of the QR factorisation of an N(0, 1) matrix, in float64,
    stored as float32;
  * LAS clip c_{t,l} ~ U[0.7, 1.0] (float32).

Rows are drawn in blocks of ``ROW_BLOCK`` tokens, each from its own
``numpy.random.default_rng([seed, module, block])`` stream, so any row can be
regenerated on its own.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np

ROW_BLOCK = 256

# stream tags: keep every draw in its own numpy stream
_TAG_ACT, _TAG_OUTLIER, _TAG_W, _TAG_P1, _TAG_P2, _TAG_LAS = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Linear:
    """One shared linear of the looped block: y = x W^T with W of shape N x K."""
    name: str
    K: int
    N: int
    a: int  # K = a * b; P1 is a x a, P2 is b x b
    b: int
    input_key: int  # modules that read the same hidden state share this key


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    T: int
    linears: Tuple[Linear, ...]
    a_bits: int
    outlier_frac: float
    outlier_mult: float
    x_dtype: str  # "f32" or "bf16"
    seed: int = 0
    description: str = ""


def _attn(n):
    return Linear(n, 2048, 2048, 32, 64, 0 if n in ("q", "k", "v") else 1)


TINY = Workload(
    "tiny", M=64, T=4,
    linears=(Linear("shared", 256, 256, 16, 16, 0),),
    a_bits=4, outlier_frac=0.02, outlier_mult=20.0, x_dtype="f32",
    description="one shared linear K=N=256, M=64, T=4, W4A4 g32, fp32 x, "
                "16x16 (x) 16x16 Kronecker factors")

ATTN_PROJ = Workload(
    "attn_proj_2048", M=2048, T=4,
    linears=(Linear("proj", 2048, 2048, 32, 64, 0),),
    a_bits=4, outlier_frac=0.02, outlier_mult=20.0, x_dtype="bf16",
    description="Ouro-1.4B-shaped attention projection K=N=2048, M=8x256 "
                "tokens, T=4, W4A4 g32, 32x32 (x) 64x64, bf16 x")

MLP = Workload(
    "mlp_2048_5632", M=2048, T=4,
    linears=(Linear("gate", 2048, 5632, 32, 64, 0),
             Linear("up", 2048, 5632, 32, 64, 0),
             Linear("down", 5632, 2048, 64, 88, 1)),
    a_bits=4, outlier_frac=0.01, outlier_mult=30.0, x_dtype="bf16",
    description="Ouro-1.4B-shaped MLP gate/up 2048->5632, down 5632->2048, "
                "M=2048, T=4, W4A4 g32, bf16 x")

CALIB_BLOCK = Workload(
    "calib_block_262144", M=262144, T=4,
    linears=(_attn("q"), _attn("k"), _attn("v"), _attn("o"),
             Linear("gate", 2048, 5632, 32, 64, 2),
             Linear("up", 2048, 5632, 32, 64, 2),
             Linear("down", 5632, 2048, 64, 88, 3)),
    a_bits=4, outlier_frac=0.02, outlier_mult=20.0, x_dtype="bf16",
    description="7 shared linears x T=4 loops on M=1024x256 tokens, W4A4 g32")


def decode_workload(M: int, N: int, a_bits: int) -> Workload:
    assert M in (1, 4, 16) and N in (2048, 5632) and a_bits in (4, 8)
    return Workload(
        f"decode_M{M}_N{N}_W4A{a_bits}", M=M, T=4,
        linears=(Linear("dec", 2048, N, 32, 64, 0),),
        a_bits=a_bits, outlier_frac=0.02, outlier_mult=20.0, x_dtype="bf16",
        description=f"decode M={M}, K=2048, N={N}, T=4, W4A{a_bits}")


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng([seed, *key])


def outlier_channels(K: int, frac: float, seed: int, input_key: int) -> np.ndarray:
    """Indices of the outlier channels of one hidden state (fixed across tokens and loops)."""
    n = int(round(frac * K))
    return np.sort(_rng(seed, _TAG_OUTLIER, input_key, K).choice(K, n, replace=False))


def base_rows(K: int, rows: Sequence[int] | np.ndarray, *, frac: float, mult: float,
              seed: int, input_key: int) -> np.ndarray:
    """Base activation x (before loop drift) for the given token rows, float32."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, K), dtype=np.float32)
    blocks = rows // ROW_BLOCK
    for blk in np.unique(blocks):
        sel = np.nonzero(blocks == blk)[0]
        full = _rng(seed, _TAG_ACT, input_key, K, int(blk)).standard_normal((ROW_BLOCK, K))
        out[sel] = full[rows[sel] - blk * ROW_BLOCK].astype(np.float32)
    ch = outlier_channels(K, frac, seed, input_key)
    out[:, ch] *= np.float32(mult)
    return out


def base_activation(M: int, K: int, *, frac: float, mult: float, seed: int,
                    input_key: int) -> np.ndarray:
    return base_rows(K, np.arange(M), frac=frac, mult=mult, seed=seed, input_key=input_key)


def drift(x: np.ndarray, t: int) -> np.ndarray:
    """x_t = fl32(fl32((1 + 0.25 t) x) + fl32(0.1 t)) in float32."""
    x = np.asarray(x, dtype=np.float32)
    mul = np.float32(1.0 + 0.25 * t)
    add = np.float32(0.1 * t)
    return (x * mul) + add


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bfloat16 (ties to even); returned as float32 values."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def bf16_bits(x_bf16_valued: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exactly bfloat16."""
    u = np.asarray(x_bf16_valued, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value is not a bfloat16"
    return (u >> 16).astype(np.uint16)


def loop_input(wl: Workload, lin: Linear, t: int, rows=None) -> np.ndarray:
    """Input x_{t,l} of linear ``lin`` at loop t (float32 values; bf16-exact for bf16 workloads)."""
    rows = np.arange(wl.M) if rows is None else rows
    x = base_rows(lin.K, rows, frac=wl.outlier_frac, mult=wl.outlier_mult,
                  seed=wl.seed, input_key=lin.input_key)
    x = drift(x, t)
    if wl.x_dtype == "bf16":
        x = round_bf16(x)
    return x


def weight(N: int, K: int, seed: int, module: int) -> np.ndarray:
    return (_rng(seed, _TAG_W, module, N, K).standard_normal((N, K)) * 0.02).astype(np.float32)


def orthogonal(n: int, seed: int, module: int, which: int) -> np.ndarray:
    tag = _TAG_P1 if which == 1 else _TAG_P2
    g = _rng(seed, tag, module, n).standard_normal((n, n))
    q, _ = np.linalg.qr(g)
    return q.astype(np.float32)


def las(T: int, seed: int, module: int) -> np.ndarray:
    return _rng(seed, _TAG_LAS, module, T).uniform(0.7, 1.0, size=T).astype(np.float32)


@dataclass
class ModuleParams:
    lin: Linear
    W: np.ndarray     # N x K float32, original (unfolded) weight
    P1: np.ndarray    # a x a float32
    P2: np.ndarray    # b x b float32
    las: np.ndarray   # [T] float32


def module_params(wl: Workload) -> List[ModuleParams]:
    out = []
    for l, lin in enumerate(wl.linears):
        out.append(ModuleParams(
            lin=lin,
            W=weight(lin.N, lin.K, wl.seed, l),
            P1=orthogonal(lin.a, wl.seed, l, 1),
            P2=orthogonal(lin.b, wl.seed, l, 2),
            las=las(wl.T, wl.seed, l)))
    return out


def device_loop_input(wl: Workload, lin: Linear, t: int, device="cuda"):
    """Large-workload variant of ``loop_input`` drawn on the device with torch's
    generator (same recipe, different random stream).  Tests copy the rows
    they check back to the host and feed those to the oracle."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([wl.seed, _TAG_ACT, lin.input_key,
                                              lin.K]).generate_state(1)[0]))
    x = torch.randn((wl.M, lin.K), generator=g, device=device, dtype=torch.float32)
    ch = torch.from_numpy(outlier_channels(lin.K, wl.outlier_frac, wl.seed, lin.input_key))
    x[:, ch.to(device)] *= torch.tensor(wl.outlier_mult, dtype=torch.float32, device=device)
    x = x * torch.tensor(1.0 + 0.25 * t, dtype=torch.float32, device=device)
    x = x + torch.tensor(float(np.float32(0.1 * t)), dtype=torch.float32, device=device)
    return x.to(torch.bfloat16) if wl.x_dtype == "bf16" else x


def random_uniform(shape, lo: float, hi: float, seed: int, *key: int) -> np.ndarray:
    return _rng(seed, 99, *key).uniform(lo, hi, size=shape).astype(np.float32)


def random_normal(shape, seed: int, *key: int, scale: float = 1.0) -> np.ndarray:
    return (_rng(seed, 98, *key).standard_normal(shape) * scale).astype(np.float32)
