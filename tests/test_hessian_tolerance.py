"""The Hessian parity rule (tests.parity.check_hessian) has the power to catch
what it must: planted mistakes in a float64 oracle result fail it, on the CPU.

  * a 64-row chunk of one loop left out of the sum (a dropped TMA stage);
  * the whole 8192-row reduction in one float32 accumulator that truncates
    once per 16-term MMA (the accumulation error the sliced kernel removes);
while the oracle's own result rounded once to float32, and the same
truncating accumulation run slice by slice with the partial sums added in
float32 (what the kernel does), pass."""
import numpy as np
import pytest

from bit_ptq_looped_b200 import synth
from oracle import lq_oracle as O
from tests.parity import HESSIAN_SLICE_ROWS, check_hessian


def _inputs(M, K, T, seed=3):
    rng = np.random.default_rng(seed)
    xs = []
    for t in range(T):
        x = rng.standard_normal((M, K)).astype(np.float32)
        x[:, rng.choice(K, max(1, K // 50), replace=False)] *= 20.0
        xs.append(synth.round_bf16((1 + 0.25 * t) * x + 0.1 * t))
    return xs


def _f32_toward_zero(v):
    """float64 values rounded to float32 toward zero."""
    f = v.astype(np.float32)
    over = np.abs(f.astype(np.float64)) > np.abs(v)
    f[over] = np.nextafter(f[over], np.float32(0))
    return f


def _truncating_sum(X, rows):
    """sum over `rows` of X[r]^T X[r], 16 rows per step, each step's exact sum
    added to a float32 accumulator that truncates."""
    K = X.shape[1]
    acc = np.zeros((K, K), np.float32)
    for r0 in range(rows.start, rows.stop, 16):
        blk = X[r0:min(r0 + 16, rows.stop)].astype(np.float64)
        acc = _f32_toward_zero(acc.astype(np.float64) + blk.T @ blk)
    return acc


@pytest.fixture(scope="module")
def case():
    M, K, T = 2048, 128, 4
    xs = _inputs(M, K, T)
    Hor = O.trajectory_hessian(xs)
    A = O.trajectory_hessian([np.abs(x) for x in xs])
    return xs, Hor, A, M * T


def test_oracle_rounded_once_passes(case):
    xs, Hor, A, n = case
    check_hessian(Hor.astype(np.float32), Hor, A, n)


def test_dropped_chunk_fails(case):
    xs, Hor, A, n = case
    bad = [x.copy() for x in xs]
    bad[1][640:704] = 0  # rows 640..703 of loop 1 never reach the sum
    with pytest.raises(AssertionError):
        check_hessian(O.trajectory_hessian(bad).astype(np.float32), Hor, A, n)


def test_single_truncating_accumulator_fails(case):
    xs, Hor, A, n = case
    X = np.concatenate(xs)
    with pytest.raises(AssertionError):
        check_hessian(_truncating_sum(X, range(0, n)), Hor, A, n)


def test_sliced_truncating_accumulators_pass(case):
    xs, Hor, A, n = case
    X = np.concatenate(xs)
    H = np.zeros_like(Hor, dtype=np.float32)
    for r0 in range(0, n, HESSIAN_SLICE_ROWS):
        H = (H + _truncating_sum(X, range(r0, min(r0 + HESSIAN_SLICE_ROWS, n)))).astype(np.float32)
    check_hessian(H, Hor, A, n)
