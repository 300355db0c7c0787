"""CPU oracle for the LoopQ-style quantized looped linear.  TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run this module.  The
library never does: it shares no code, header, table or helper with it.

This is a plain, slow, step-by-step restatement of what the pages define, in
numpy.  Each function names the passage it follows.  Sources:

* "paper_specification.yaml" of the LoopQ reproduction (page
  loopq_quantization/scripts/configs/paper_specification.yaml):
  - lq1_quantization.equation: Section 2, Eq. (4),
    Q_a(x; c) = c * clip(round(x / c), q_min, q_max);
  - lq1_quantization.method: Section 5.1, symmetric uniform RTN;
  - lq1_quantization.granularity: Section 5.1 / Appendix B.3 Table 6,
    weights and activations group-wise, group size 32;
  - lq1_quantization.evaluated_precisions: W4 with A4 or A8;
  - loopq_components.las: Section 4.1, one clip c_{t,l} per module and loop;
  - implementation_status.lq2: positive per-module/per-loop clipping scalars
    applied to dynamic token/group absmax scales;
  - loopq_components.shared_transformed_backbone: Section 2, Eqs. (2)-(3),
    an invertible P_l folded into activation and weight sides;
  - implementation_status.lq3: shared Kronecker transform and exact no-quant
    inverse-transpose weight folding;
  - paper_underspecified_items: integer bounds, tie-breaking, initial scale
    estimator, group axis/tail, epsilons and the Kronecker details are not
    fixed by the paper.
* LoopQ reproduction README ("LoopQ 4-bit quantization of Ouro-1.4B"):
  header (24 layers run 4 times per token), arm table
  (rtn_w4a4_group32, rtn_w4a4_per_token, loopq_w4a4_untrained = random
  orthogonal Kronecker transforms with LAS clip 1.0).

Readings taken where the pages are silent (each is pinned by a test):
  integer bounds q_min = -q_max, q_max = 2^(bits-1) - 1 (-7..7, -127..127);
  round half to even; step s = fl32(fl32(c * absmax) / q_max) from the dynamic
  group absmax (weights: c = 1); codes q = clip(rne(fl32(x / s))) and q = 0
  for an all-zero group (no epsilon); groups of 32 consecutive elements along K
  (the contraction axis), K a multiple of 32, no tail; the Kronecker transform
  acts on a token row as x (P1 kron P2), i.e. on the row-major a x b reshape X
  as P1^T X P2, computed in float64 and rounded once to float32; weights are
  folded as W (P1^-T kron P2^-T); int4 codes are packed two per byte, even
  element in bits 3..0, odd element in bits 7..4, two's complement; the GEMM
  sums q_a q_w exactly per group and rescales by s_a s_w in float64.

All float32 steps use numpy float32 scalar/array arithmetic, which is IEEE
single precision with round-to-nearest-even and no fused multiply-add.
"""
from __future__ import annotations

import numpy as np

GROUP = 32


def qmax_for_bits(bits: int) -> int:
    """q_max = 2^(bits-1) - 1 (reading of the unspecified integer bounds: symmetric)."""
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8 (Section 5.1 evaluated precisions)")
    return (1 << (bits - 1)) - 1


# --------------------------------------------------------------------------
# Kronecker transform (shared transformed backbone, Section 2 Eqs. (2)-(3);
# implementation_status.lq3)
# --------------------------------------------------------------------------
def kron_rotate_f64(x: np.ndarray, P1: np.ndarray, P2: np.ndarray) -> np.ndarray:
    """x (P1 kron P2) for every row of x in float64 (not rounded).

    With the row-major reshape X = x.reshape(a, b) (index k = i*b + j), the
    product x (P1 kron P2) equals vec(P1^T X P2).
    """
    x = np.asarray(x, dtype=np.float64)
    a, b = P1.shape[0], P2.shape[0]
    M, K = x.shape
    assert K == a * b
    X = x.reshape(M, a, b)
    Z = np.einsum("pi,mpq,qj->mij", np.asarray(P1, np.float64), X,
                  np.asarray(P2, np.float64), optimize=True)
    return Z.reshape(M, K)


def kron_rotate(x: np.ndarray, P1: np.ndarray, P2: np.ndarray) -> np.ndarray:
    """x~ = x (P1 kron P2): float64 arithmetic, rounded once to float32."""
    return kron_rotate_f64(x, P1, P2).astype(np.float32)


def kron_rotate_dense(x: np.ndarray, P1: np.ndarray, P2: np.ndarray) -> np.ndarray:
    """Same transform through the dense K x K Kronecker matrix (small K only)."""
    P = np.kron(np.asarray(P1, np.float64), np.asarray(P2, np.float64))
    return (np.asarray(x, np.float64) @ P).astype(np.float32)


def inverse_transpose(P: np.ndarray) -> np.ndarray:
    """P^{-T} in float64 (the weight-side factor of the fold)."""
    return np.linalg.inv(np.asarray(P, np.float64)).T


def fold_weights(W: np.ndarray, Q1: np.ndarray, Q2: np.ndarray) -> np.ndarray:
    """W~ = W (Q1 kron Q2), float64 arithmetic, rounded once to float32.

    Callers pass Q = P^{-T} (inverse-transpose folding, implementation_status.lq3);
    for orthogonal P this is P itself, so x~ W~^T = x W^T without quantization.
    """
    return kron_rotate(W, Q1, Q2)


# --------------------------------------------------------------------------
# Quantizer Q_a (Section 2 Eq. (4), Section 5.1 RTN, group 32, LAS Section 4.1)
# --------------------------------------------------------------------------
def quantize_groups(xt: np.ndarray, c: float, bits: int, group: int = GROUP):
    """Symmetric group RTN of a float32 matrix.

    For every row m and group g of ``group`` consecutive elements along K:
      absmax = max |x~|            (dynamic group absmax)
      s      = fl32(fl32(c * absmax) / q_max)   (LAS clip c on the absmax scale)
      q      = clip(rne(fl32(x~ / s)), -q_max, q_max),   q = 0 where s == 0.
    Returns (codes int8 M x K, scales float32 M x G).
    """
    xt = np.asarray(xt, dtype=np.float32)
    M, K = xt.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    if not (c > 0):
        raise ValueError("LAS clip must be positive")
    qmax = qmax_for_bits(bits)
    G = K // group
    xg = xt.reshape(M, G, group)
    amax = np.abs(xg).max(axis=2)                         # float32, exact
    s = (np.float32(c) * amax) / np.float32(qmax)         # two float32 roundings
    with np.errstate(divide="ignore", invalid="ignore"):
        r = xg / s[:, :, None]                            # float32 division
    q = np.rint(r)                                        # round half to even
    q = np.clip(q, -qmax, qmax)
    q = np.where(s[:, :, None] == 0, 0.0, q)
    return q.astype(np.int8).reshape(M, K), s.astype(np.float32)


def quantize_weights(Wt: np.ndarray, group: int = GROUP):
    """Weight RTN (4-bit, group 32 along K): s_w = fl32(absmax / 7), no clip scalar."""
    return quantize_groups(Wt, 1.0, 4, group)


def quantize_activation(x: np.ndarray, P1, P2, c: float, bits: int, group: int = GROUP):
    """Rotate (if P1/P2 given) then quantize one activation matrix."""
    xt = kron_rotate(x, P1, P2) if P1 is not None else np.asarray(x, np.float32)
    return quantize_groups(xt, c, bits, group)


# --------------------------------------------------------------------------
# int4 packing (storage format of 4-bit codes)
# --------------------------------------------------------------------------
def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element 2j in bits 3..0, element 2j+1 in bits 7..4 (two's complement)."""
    q = np.asarray(codes, dtype=np.int64)
    assert q.shape[-1] % 2 == 0
    assert np.all((q >= -8) & (q <= 7))
    nib = (q & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# --------------------------------------------------------------------------
# Group-rescaled integer GEMM
# --------------------------------------------------------------------------
def group_gemm(qa: np.ndarray, sa: np.ndarray, qw: np.ndarray, sw: np.ndarray,
               group: int = GROUP) -> np.ndarray:
    """y[m,n] = sum_g sa[m,g] sw[n,g] sum_{k in g} qa[m,k] qw[n,k], in float64.

    The per-group integer sums are formed with a float64 matmul of the integer
    codes: every product and partial sum is an integer below 2^15 in magnitude,
    so they are exact in float64 whatever order the library sums them in.
    """
    qa = np.asarray(qa)
    qw = np.asarray(qw)
    M, K = qa.shape
    N = qw.shape[0]
    assert qw.shape[1] == K and K % group == 0
    G = K // group
    sa = np.asarray(sa, np.float64)
    sw = np.asarray(sw, np.float64)
    y = np.zeros((M, N), dtype=np.float64)
    for g in range(G):
        ka = qa[:, g * group:(g + 1) * group].astype(np.float64)
        kw = qw[:, g * group:(g + 1) * group].astype(np.float64)
        acc = ka @ kw.T
        y += (sa[:, g][:, None] * sw[:, g][None, :]) * acc
    return y


# --------------------------------------------------------------------------
# Loop driver (README header: the shared layers run 4 times per token;
# loopq_components.las: c_{t,l} per module and loop)
# --------------------------------------------------------------------------
class OracleLayer:
    """One shared quantized linear: folded + quantized weights, its P factors and LAS clips."""

    def __init__(self, W: np.ndarray, P1: np.ndarray, P2: np.ndarray, las: np.ndarray,
                 a_bits: int, group: int = GROUP, fold: bool = True, Q1=None, Q2=None):
        """Q1, Q2: the weight-side fold factors; by default P^{-T} rounded to
        float32, the form in which a float32 library receives them."""
        self.P1 = np.asarray(P1, np.float32)
        self.P2 = np.asarray(P2, np.float32)
        self.las = np.asarray(las, np.float32)
        self.a_bits = a_bits
        self.group = group
        if fold:
            self.Q1 = inverse_transpose(self.P1).astype(np.float32) if Q1 is None else Q1
            self.Q2 = inverse_transpose(self.P2).astype(np.float32) if Q2 is None else Q2
            self.W_folded64 = kron_rotate_f64(W, self.Q1, self.Q2)
            Wt = self.W_folded64.astype(np.float32)
        else:
            Wt = np.asarray(W, np.float32)
            self.W_folded64 = Wt.astype(np.float64)
        self.W_folded = Wt
        self.qw, self.sw = quantize_weights(Wt, group)
        self.N, self.K = Wt.shape

    def forward(self, x: np.ndarray, t: int) -> np.ndarray:
        if not (0 <= t < self.las.size):
            raise ValueError("loop index out of range")
        qa, sa = quantize_activation(x, self.P1, self.P2, float(self.las[t]), self.a_bits,
                                     self.group)
        return group_gemm(qa, sa, self.qw, self.sw, self.group)


def loop_linear(x: np.ndarray, layer: OracleLayer, t: int) -> np.ndarray:
    return layer.forward(x, t)


def loop_stack_open(xs, layers, T: int):
    """Open mode: input xs[t][l] for every loop t and layer l; returns ys[t][l] (float64)."""
    return [[loop_linear(xs[t][l], layers[l], t) for l in range(len(layers))]
            for t in range(T)]


def loop_stack_chain(x0: np.ndarray, layers, T: int):
    """Chain mode: y_{t,l} is the input of the next step; the library carries it in float32."""
    ys = []
    cur = np.asarray(x0, np.float32)
    for t in range(T):
        row = []
        for l, layer in enumerate(layers):
            y = loop_linear(cur, layer, t)
            row.append(y)
            cur = y.astype(np.float32)
        ys.append(row)
    return ys


def loop_stack_slt_open(xs, layers_tl, T: int):
    """SLT serving ("paper_specification.yaml" of the LoopQ reproduction: slt,
    Section 4.2, Eqs. (5)-(6)): the modules SLT selected carry a loop-dependent
    transform and weight, so step (t, l) applies its own layer layers_tl[t][l];
    the others repeat their shared layer.  Open mode: input xs[t][l]."""
    return [[loop_linear(xs[t][l], layers_tl[t][l], t) for l in range(len(layers_tl[t]))]
            for t in range(T)]


def loop_stack_slt_chain(x0: np.ndarray, layers_tl, T: int):
    """SLT serving in chain mode: y_{t,l} (carried in float32) feeds step (t, l+1)."""
    ys = []
    cur = np.asarray(x0, np.float32)
    for t in range(T):
        row = []
        for layer in layers_tl[t]:
            y = loop_linear(cur, layer, t)
            row.append(y)
            cur = y.astype(np.float32)
        ys.append(row)
    return ys


# ----------------------------------------------------------------------------
# cross-loop transition alignment (CTA) at loop transitions
# ----------------------------------------------------------------------------
def cta_apply(h: np.ndarray, a_t: np.ndarray, b_t: np.ndarray, eta_t: float,
              U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """CTA ("paper_specification.yaml" of the LoopQ reproduction: cta, Section
    4.3, Eq. (7); implementation_status lq5): an affine plus gated low-rank
    adapter applied only at loop transitions, U and V shared across
    transitions, a_t, b_t and the gate eta_t loop-dependent; rank 8
    (cta_rank); identity at initialization.  Eq. (7) itself is not printed on
    the pages; the plainest reading of that description is taken:

        h' = a_t * h + b_t + eta_t * (h V) U^T      (U, V: d x r; a_t, b_t: d)

    computed in float64 and rounded once to float32 (the carried state is
    float32)."""
    h64 = np.asarray(h, np.float32).astype(np.float64)
    p = h64 @ np.asarray(V, np.float32).astype(np.float64)            # M x r
    low = p @ np.asarray(U, np.float32).astype(np.float64).T          # M x d
    out = (np.asarray(a_t, np.float32).astype(np.float64)[None, :] * h64
           + np.asarray(b_t, np.float32).astype(np.float64)[None, :]
           + np.float64(np.float32(eta_t)) * low)
    return out.astype(np.float32)


def loop_stack_chain_cta(x0: np.ndarray, layers, T: int, a, b, eta, U, V):
    """Chain mode with CTA at every transition: after loop t < T - 1 the state
    that feeds loop t + 1 is cta_apply(y_{t, L-1}, a[t], b[t], eta[t]); the
    outputs y_{t,l} themselves are returned unadapted."""
    ys = []
    cur = np.asarray(x0, np.float32)
    for t in range(T):
        row = []
        for layer in layers:
            y = loop_linear(cur, layer, t)
            row.append(y)
            cur = y.astype(np.float32)
        if t + 1 < T:
            cur = cta_apply(cur, a[t], b[t], eta[t], U, V)
        ys.append(row)
    return ys


# ----------------------------------------------------------------------------
# trajectory Hessian accumulation (calibration statistic)
# ----------------------------------------------------------------------------
def trajectory_hessian(xs) -> np.ndarray:
    """H = sum_t X_t^T X_t over the inputs X_t (M x K) a module sees at each
    loop t ("Quantizing Looped Transformers: Feedback Exposure and Calibration
    Blindness", Appendix Table 19: H_t = X_t^T X_t per recurrence step;
    abstract and Section 5: accumulating the GPTQ Hessian across recurrence
    steps instead of the step-0 activations alone).  Unnormalised (the
    row-normalised form of Figure 5, 2 X^T X / m, is a scalar multiple);
    float64."""
    K = np.asarray(xs[0]).shape[1]
    H = np.zeros((K, K), np.float64)
    for x in xs:
        x64 = np.asarray(x, np.float32).astype(np.float64)
        H += x64.T @ x64
    return H

