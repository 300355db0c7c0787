"""GPU parity of the trajectory Hessian H = sum_t X_t^T X_t (lq_trajectory_hessian)
against the CPU oracle."""
import numpy as np
import pytest
import torch

from bit_ptq_looped_b200 import lq, synth
from oracle import lq_oracle as O
from tests.parity import check_hessian, dev, host

pytestmark = pytest.mark.gpu


def _inputs(M, K, T, seed):
    rng = np.random.default_rng(seed)
    xs = []
    for t in range(T):
        x = rng.standard_normal((M, K)).astype(np.float32)
        ch = rng.choice(K, max(1, K // 50), replace=False)
        x[:, ch] *= 20.0  # outlier channels, as in the configs' activations
        xs.append(synth.round_bf16((1 + 0.25 * t) * x + 0.1 * t))
    return xs


def _bf16_device(xs):
    flat = np.concatenate([x.ravel() for x in xs])
    return torch.from_numpy(flat).to(torch.bfloat16).cuda()


def _check(Hg, xs, H0=None, rows=None):
    """Against the float64 oracle, within the bound of the kernel's summation
    (tests.parity.check_hessian): relative Frobenius error <= 1e-5 and every
    element within that bound."""
    n = sum(x.shape[0] for x in xs)
    if rows is None:
        Hor = O.trajectory_hessian(xs)
        A = O.trajectory_hessian([np.abs(x) for x in xs])
    else:
        Hor = sum(x[:, rows].astype(np.float64).T @ x.astype(np.float64) for x in xs)
        A = sum(np.abs(x[:, rows]).astype(np.float64).T @ np.abs(x).astype(np.float64) for x in xs)
        Hg = Hg[rows]
        H0 = None if H0 is None else H0[rows]
    if H0 is not None:
        Hor = Hor + H0
        A = A + np.abs(H0)
    return check_hessian(Hg, Hor, A, n)


@pytest.mark.parametrize("M,K,T", [(64, 256, 4), (1024, 1024, 2), (100, 384, 3), (1, 128, 1)])
def test_trajectory_hessian_matches_oracle(M, K, T):
    xs = _inputs(M, K, T, seed=M + K + T)
    H = host(lq.lq_trajectory_hessian(_bf16_device(xs), T, M=M))
    torch.cuda.synchronize()
    assert np.array_equal(H, H.T)  # the lower triangle is the mirrored upper one
    _check(H, xs)


def test_trajectory_hessian_accumulates():
    M, K, T = 300, 512, 2
    xs = _inputs(M, K, T, seed=9)
    H0 = np.random.default_rng(1).standard_normal((K, K)).astype(np.float32)
    H0 = (H0 + H0.T) / 2
    Hd = dev(H0)
    lq.lq_trajectory_hessian(_bf16_device(xs), T, M=M, H=Hd, accumulate=True)
    torch.cuda.synchronize()
    _check(host(Hd), xs, H0=H0.astype(np.float64))


def test_trajectory_hessian_full_size_sampled_rows():
    """attn_proj-shaped loop inputs: M = 2048 tokens, K = 2048, T = 4 loops
    (a reduction of 8192 rows, 32 accumulator slices); 16 sampled rows of H
    against the oracle."""
    M, K, T = 2048, 2048, 4
    xs = _inputs(M, K, T, seed=21)
    H = host(lq.lq_trajectory_hessian(_bf16_device(xs), T, M=M))
    torch.cuda.synchronize()
    rows = np.random.default_rng(2).choice(K, 16, replace=False)
    _check(H, xs, rows=rows)


def test_trajectory_hessian_rejects_bad_calls():
    x = torch.zeros(64 * 200, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lq.LQError) as e:  # K not a multiple of 128
        lq.lq_trajectory_hessian(x.view(64, 200), 1, M=64)
    assert e.value.status == lq.LQ_ERR_SHAPE
    with pytest.raises(lq.LQError) as e:
        lq.lq_trajectory_hessian(torch.zeros((64, 256), device="cuda"), 1, M=64)
    assert e.value.status == lq.LQ_ERR_UNSUPPORTED
