"""Why the Kronecker rotation runs on the FP64 tensor-core MMA and not on a
split-precision bf16 / fp16 tensor-core product (measured, on the CPU).

The fused rotate+quantize rule lets a code differ from the oracle's only where
the oracle's x~/s lies within 1e-6 (relative) of a rounding tie.  A rotation
whose error moves x~/s by more than that window anywhere can flip codes
outside it whenever x~/s falls between the window and the error, which at the
workloads' sizes (millions of codes per step) is expected to happen.  The
candidate split forms are emulated here exactly as a tensor core would run
them: each float32 factor cut into bf16 (3 pieces) or fp16 (2 pieces), exact
products, float32 accumulation per 16-wide K chunk, rounded to nearest (the
best case) or truncated; the second stage splits the float32 intermediate the
same way.  On attention- and MLP-shaped rows the error exceeds the window on
a sizeable fraction of the codes, so the split forms cannot meet the rule; the
float64 accumulation the kernel uses stays many orders of magnitude inside it.
"""
import numpy as np
import pytest

from bit_ptq_looped_b200 import synth
from oracle import lq_oracle as O


def _round_bits(v, bits):
    m, e = np.frexp(v)
    return np.ldexp(np.round(m * 2.0 ** bits) / 2.0 ** bits, e)


def _split(v, bits, n):
    out, r = [], np.asarray(v, np.float64)
    for _ in range(n):
        p = _round_bits(r, bits)
        out.append(p)
        r = r - p
    return out


def _f32(v, mode):
    f = v.astype(np.float32)
    if mode == "rz":
        over = np.abs(f.astype(np.float64)) > np.abs(v)
        f[over] = np.nextafter(f[over], np.float32(0))
    return f.astype(np.float64)


def _rotate_split(x, P1, P2, bits, n, mode):
    """x (P1 kron P2) as vec(P1^T X P2) from split pieces, float32 accumulation
    per 16-wide K chunk (pieces i + j < n of the second-stage products)."""
    M, K = x.shape
    a, b = P1.shape[0], P2.shape[0]
    X = x.astype(np.float64).reshape(M, a, b)
    acc = None
    for p in _split(P2, bits, n):  # stage 1: Y = X P2 (x exact in bf16)
        for k0 in range(0, b, 16):
            part = X[..., k0:k0 + 16] @ p[k0:k0 + 16]
            acc = _f32(part if acc is None else acc + part, mode)
    p1s, ys = _split(np.asarray(P1, np.float64).T, bits, n), _split(acc, bits, n)
    acc = None
    for i in range(n):  # stage 2: Z = P1^T Y
        for j in range(n - i):
            for k0 in range(0, a, 16):
                part = np.einsum("ip,mpj->mij", p1s[i][:, k0:k0 + 16], ys[j][:, k0:k0 + 16, :])
                acc = _f32(part if acc is None else acc + part, mode)
    return acc.reshape(M, K)


def _window_ratio(wl, li, rows, rotate):
    lin, mp = wl.linears[li], synth.module_params(wl)[li]
    x = synth.loop_input(wl, lin, 1, rows=np.arange(rows))
    xt64 = O.kron_rotate_f64(x, mp.P1, mp.P2)
    _, s = O.quantize_groups(xt64.astype(np.float32), float(mp.las[1]), wl.a_bits)
    s = s.astype(np.float64)[:, :, None]
    r = (xt64.reshape(rows, -1, 32) / s).reshape(rows, -1)
    window = 1e-6 * (np.floor(np.abs(r)) + 0.5)
    dr = (np.abs(rotate(x, mp.P1, mp.P2) - xt64).reshape(rows, -1, 32) / s).reshape(rows, -1)
    return dr / window


@pytest.mark.parametrize("wl,li", [(synth.ATTN_PROJ, 0), (synth.MLP, 2)], ids=["attn", "mlp_down"])
@pytest.mark.parametrize("bits,n", [(8, 3), (11, 2)], ids=["bf16x3", "fp16x2"])
def test_split_precision_rotation_leaves_the_tie_window(wl, li, bits, n):
    ratio = _window_ratio(wl, li, 32, lambda x, P1, P2: _rotate_split(x, P1, P2, bits, n, "rn"))
    # even with round-to-nearest accumulation the error passes the window on
    # more than 0.1 % of the codes, by more than twice the window
    assert (ratio > 1).mean() > 1e-3 and ratio.max() > 2


@pytest.mark.parametrize("wl,li", [(synth.ATTN_PROJ, 0), (synth.MLP, 2)], ids=["attn", "mlp_down"])
def test_float64_accumulation_stays_inside_the_tie_window(wl, li):
    """The kernel's form: float64 products and sums of the float32 factors,
    rounded once to float32; here without that final rounding (the oracle
    rounds the same value), in another summation order than the oracle's."""
    def rot(x, P1, P2):
        X = x.astype(np.float64).reshape(len(x), P1.shape[0], P2.shape[0])
        Y = X @ np.asarray(P2, np.float64)
        return np.einsum("pi,mpj->mij", np.asarray(P1, np.float64), Y).reshape(len(x), -1)
    assert _window_ratio(wl, li, 32, rot).max() < 1e-6
