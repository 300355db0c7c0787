"""Comparison rules shared by the GPU parity tests (CUDA path vs the CPU oracle).

Tolerances (stated for the quantized looped linear):
  * quantizer fed the same float32 transformed input: codes and steps bit-exact;
  * fused rotate + quantize: steps within 1e-6 relative; at most 1e-4 of the
    codes may differ, each by +-1 and only where the float64 transformed value
    divided by the step lies within 1e-6 (relative) of a rounding tie k + 1/2;
  * GEMM: max|dy| <= 1e-3 max|y| and relative L2 <= 1e-5 against the float64
    oracle, on rows whose codes agree; rows holding an allowed near-tie code
    difference are checked against the bound that difference implies;
  * trajectory Hessian (bf16 inputs, products exact in float32): relative
    Frobenius error <= 1e-5 of ||H||, and every element within the bound of
    the kernel's summation (see check_hessian).
"""
import numpy as np
import torch

from oracle import lq_oracle as O


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def act_tensor(x_f32: np.ndarray, x_dtype: str) -> torch.Tensor:
    """float32 values (bf16-exact for bf16 workloads) -> device tensor of that dtype."""
    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32))
    if x_dtype == "bf16":
        t = t.to(torch.bfloat16)
        assert torch.equal(t.float(), torch.from_numpy(np.asarray(x_f32, np.float32)))
    return t.cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def check_codes_near_tie(q_gpu, s_gpu, q_or, s_or, xt64, *, frac_max=1e-4, rel_tie=1e-6,
                         group=32):
    """Fused-path rule; returns the (row, col) indices of the allowed mismatches."""
    q_gpu = np.asarray(q_gpu, np.int64)
    q_or = np.asarray(q_or, np.int64)
    s_gpu = np.asarray(s_gpu, np.float64)
    s_or = np.asarray(s_or, np.float64)
    zero = s_or == 0
    assert np.all(s_gpu[zero] == 0)
    rel = np.abs(s_gpu - s_or)[~zero] / s_or[~zero]
    assert rel.size == 0 or rel.max() <= 1e-6, f"step rel err {rel.max()}"
    mism = q_gpu != q_or
    if not mism.any():
        return np.zeros((0, 2), np.int64)
    assert np.abs(q_gpu - q_or)[mism].max() == 1, "code differs by more than 1"
    M, K = q_or.shape
    r = xt64.reshape(M, K // group, group) / s_or[:, :, None]
    r = r.reshape(M, K)
    tie = np.floor(r) + 0.5
    dist = np.abs(r - tie)
    ok = dist[mism] <= rel_tie * np.abs(tie[mism])
    assert ok.all(), f"{(~ok).sum()} code differences are not at near-ties " \
                     f"(max dist {dist[mism].max()})"
    assert mism.mean() <= frac_max, f"{mism.mean()} of the codes differ"
    return np.argwhere(mism)


def check_gemm(y_gpu, y_or, *, exclude_rows=None, what=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_or = np.asarray(y_or, np.float64)
    if exclude_rows is not None and len(exclude_rows):
        keep = np.ones(y_or.shape[0], bool)
        keep[np.asarray(exclude_rows)] = False
        y_gpu, y_or = y_gpu[keep], y_or[keep]
    d = y_gpu - y_or
    maxy = np.abs(y_or).max()
    assert np.abs(d).max() <= 1e-3 * maxy, f"{what} max|dy| {np.abs(d).max()} vs {1e-3 * maxy}"
    rl2 = np.linalg.norm(d) / max(np.linalg.norm(y_or), 1e-300)
    assert rl2 <= 1e-5, f"{what} rel L2 {rl2}"
    return rl2


def weight_parity(q4_gpu, s_gpu, ol):
    """Resident weights vs the oracle layer: the float64 fold rounds once to
    float32 on both sides, so codes may differ only at near-ties (same rule as
    the fused activation path).  Returns the (n, k) indices that differ."""
    q_gpu = O.unpack_int4(np.asarray(q4_gpu))
    return check_codes_near_tie(q_gpu, s_gpu, ol.qw, ol.sw, ol.W_folded64)


def linear_parity(y_gpu, x, ol, t, q_gpu, s_gpu, w_flips=None):
    """Oracle y of one quantized linear (oracle layer ``ol`` at loop t) plus the
    near-tie bookkeeping: rows with an allowed activation-code difference and
    columns with an allowed weight-code difference are checked against the
    bound that difference implies, every other entry against the GEMM tolerance."""
    y_gpu = np.asarray(y_gpu)
    c = float(ol.las[t])
    xt64 = O.kron_rotate_f64(x, ol.P1, ol.P2)
    qa, sa = O.quantize_groups(xt64.astype(np.float32), c, ol.a_bits)
    qw, sw = ol.qw, ol.sw
    flips = check_codes_near_tie(q_gpu, s_gpu, qa, sa, xt64)
    y_or = O.group_gemm(qa, sa, qw, sw)
    rows = np.unique(flips[:, 0]) if len(flips) else np.zeros(0, np.int64)
    cols = np.unique(w_flips[:, 0]) if w_flips is not None and len(w_flips) else \
        np.zeros(0, np.int64)
    keep_c = np.ones(y_or.shape[1], bool)
    keep_c[cols] = False
    check_gemm(y_gpu[:, keep_c], y_or[:, keep_c], exclude_rows=rows)
    # a +-1 code difference moves y by at most s_a s_w |other code|
    bound = np.zeros_like(y_or)
    for (m, k) in flips:
        g = k // 32
        bound[m] += sa[m, g] * sw[:, g] * np.abs(qw[:, k])
    if w_flips is not None:
        for (n, k) in w_flips:
            g = k // 32
            bound[:, n] += sa[:, g] * sw[n, g] * np.abs(qa[:, k]) * 1.0001
    tol = 1e-3 * np.abs(y_or).max()
    assert np.all(np.abs(y_gpu - y_or) <= bound + tol)
    return y_or, len(flips)


# rows per accumulator slice of the Hessian kernel and MMAs (K = 16) per slice
HESSIAN_SLICE_ROWS = 256
HESSIAN_MMAS_PER_SLICE = HESSIAN_SLICE_ROWS // 16


def hessian_bound(A, n_rows):
    """Element bound of the kernel's float32 summation of n_rows exact
    products: each slice of 256 rows is summed by the tensor core (16 MMAs;
    allowed 2^-21 of the running sum of magnitudes per MMA, four units in the
    last place, since the tensor core's accumulation does not round to
    nearest), then the n_slices partial sums (and H0 when accumulating) are
    added in float32 with round to nearest (2^-24 per addition).  A is the sum
    of |x_i x_j| (plus |H0|)."""
    n_slices = -(-n_rows // HESSIAN_SLICE_ROWS)
    return (HESSIAN_MMAS_PER_SLICE * 2.0 ** -21 + (n_slices + 2) * 2.0 ** -24) * A


def check_hessian(Hg, Hor, A, n_rows):
    """Hg (the library's H or rows of it) against the float64 oracle Hor."""
    Hg = np.asarray(Hg, np.float64)
    err = np.abs(Hg - Hor)
    bound = hessian_bound(A, n_rows)
    assert np.all(err <= bound + 1e-30), f"max err/bound {(err / (bound + 1e-300)).max()}"
    rel = np.linalg.norm(err) / max(np.linalg.norm(Hor), 1e-300)
    assert rel <= 1e-5, f"relative Frobenius error {rel}"
    return rel
