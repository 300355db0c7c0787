"""An exact integer split of the Kronecker rotation (measured, on the CPU):
the plan for moving the rotation onto the 8-bit tensor cores.

Unlike the float32-accumulating splits of `test_split_rotation_precision.py`,
an integer split accumulates no rounding error: each row of the contraction's
left operand is scaled by a power of two into (-1, 1) and cut into signed
7-bit slices (|slice| <= 127, an int8 operand), the factor likewise with one
power of two, and every slice product is an exact int32 sum (at b = 88 the
largest is 88 * 127 * 127 < 2^21).  Keeping the products whose slice indices
sum to less than D, combining them exactly (as integers, one rounding to
float64) and re-slicing the float64 intermediate for the second stage, the
only error is the dropped tail of the slices, about 128^-D of each row's
scale.  Here the emulation runs the two stages of x~ = vec(P1^T X P2) that
way on attention- and MLP-down-shaped rows and measures the error against the
1e-6 tie window of the fused rotate+quantize rule.  Measured (32 rows, the
largest error over all codes, as a fraction of the window): D = 3 (6 slice
products per stage) 580x, D = 4 (10) 5.2x, D = 5 (15) 0.036-0.049,
D = 6 (21) 0.0003, D = 7 (28) 3e-6.  So 15 products per stage meet the rule
with a 20x margin.
"""
import numpy as np
import pytest

from bit_ptq_looped_b200 import synth
from tests.test_split_rotation_precision import _window_ratio


def _slices(v, n):
    """v (float64, |v| < 1) as n signed 7-bit integer slices q_k (int64):
    v = sum_k q_k 128^-(k+1) + r with |r| < 128^-n."""
    out, r = [], np.asarray(v, np.float64)
    for _ in range(n):
        q = np.trunc(r * 128.0)
        out.append(q.astype(np.int64))
        r = r * 128.0 - q
    return out


def _row_scale(v, axis):
    """Power-of-two exponents e with |v| / 2^e < 1 along `axis` (0 for an all-zero line)."""
    m = np.max(np.abs(v), axis=axis, keepdims=True)
    _, e = np.frexp(m)
    return np.where(m > 0, e, 0)


def _int_split_matmul(A, B, D, a_axis):
    """A @ B (float64 operands) through integer slices: A scaled per line along
    the contraction (a_axis = the contraction axis of A), B by one power of
    two; the slice products with index sum < D, combined exactly."""
    ea = _row_scale(A, a_axis)
    eb = _row_scale(B, None)
    As = _slices(A / np.ldexp(1.0, ea), D)
    Bs = _slices(B / np.ldexp(1.0, eb), D)
    acc = None  # sum_{k+l<D} (A_k B_l) 128^(D-1-(k+l)), exact in int64
    for k in range(D):
        for l in range(D - k):
            term = np.matmul(As[k], Bs[l]) * (128 ** (D - 1 - k - l))
            acc = term if acc is None else acc + term
    return acc.astype(np.float64) * np.ldexp(1.0, ea + eb) / 128.0 ** (D + 1)


def _rotate_int_split(x, P1, P2, D):
    M, K = x.shape
    a, b = P1.shape[0], P2.shape[0]
    X = x.astype(np.float64).reshape(M, a, b)
    # stage 1: Y = X P2, X's rows (length b) scaled one by one
    Y = _int_split_matmul(X, np.asarray(P2, np.float64), D, a_axis=2)
    # stage 2: Z = P1^T Y, Y's columns (length a) scaled one by one
    Zt = _int_split_matmul(np.swapaxes(Y, 1, 2), np.asarray(P1, np.float64), D, a_axis=2)
    return np.swapaxes(Zt, 1, 2).reshape(M, K)


@pytest.mark.parametrize("wl,li", [(synth.ATTN_PROJ, 0), (synth.MLP, 2)], ids=["attn", "mlp_down"])
def test_int_slice_rotation_stays_inside_the_tie_window(wl, li):
    ratio = _window_ratio(wl, li, 32, lambda x, P1, P2: _rotate_int_split(x, P1, P2, 5))
    assert ratio.max() < 0.1


@pytest.mark.parametrize("wl,li", [(synth.ATTN_PROJ, 0), (synth.MLP, 2)], ids=["attn", "mlp_down"])
def test_int_slice_rotation_needs_enough_slices(wl, li):
    ratio = _window_ratio(wl, li, 32, lambda x, P1, P2: _rotate_int_split(x, P1, P2, 4))
    assert ratio.max() > 1


def test_int_slices_are_int8_and_products_fit_int32():
    rng = np.random.default_rng(3)
    v = rng.uniform(-1, 1, (64, 88)) * (1 - 1e-12)
    qs = _slices(v, 5)
    assert all(np.abs(q).max() <= 127 for q in qs)
    # a slice product over the longest contraction here (b = 88) fits in int32
    assert 88 * 127 * 127 < 2 ** 31
    # the slices reconstruct v to within 128^-5
    rec = sum(q * 128.0 ** -(k + 1) for k, q in enumerate(qs))
    assert np.max(np.abs(rec - v)) < 128.0 ** -5
