"""Pins for the CPU oracle: checks against things other than the oracle itself.

The pages print no worked example, so the pins are the hand-derived cases of
tests/golden/qa_hand_examples.json, exact-arithmetic brute force on small
inputs, closed forms and invariants of the definition, and special cases that
reduce to textbook operations.  The last tests plant mistakes in copies of
the oracle and check that some pin catches each of them.
"""
import json
import os
import types
from fractions import Fraction

import numpy as np
import pytest

from oracle import lq_oracle as O
from bit_ptq_looped_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "qa_hand_examples.json")


def _golden():
    with open(GOLD) as f:
        return json.load(f)


def _pad32(v):
    out = np.zeros((1, 32), np.float32)
    out[0, :len(v)] = np.asarray(v, np.float32)
    return out


# ----------------------------------------------------------------------------
# pin functions: each takes an oracle-like namespace so planted mistakes can be
# run through them
# ----------------------------------------------------------------------------
def pin_hand_activation(o):
    g = _golden()
    for case in g["activation_cases"]:
        q, s = o.quantize_groups(_pad32(case["x"]), case["c"], case["bits"])
        n = len(case["x"])
        if "scale" in case:
            exp_s = np.float32(case["scale"])
        else:  # fl32(2.25/7)
            exp_s = np.float32(np.float32(2.25) / np.float32(7))
        assert s[0, 0] == exp_s, case["name"]
        assert list(q[0, :n]) == case["codes"], case["name"]
        assert np.all(q[0, n:] == 0)


def pin_hand_weight(o):
    for case in _golden()["weight_cases"]:
        q, s = o.quantize_weights(_pad32(case["w"]))
        n = len(case["w"])
        assert s[0, 0] == np.float32(case["scale"])
        assert list(q[0, :n]) == case["codes"]


def pin_hand_packing(o):
    for case in _golden()["packing_cases"]:
        b = o.pack_int4(np.asarray([case["codes"]], np.int8))
        assert list(b[0]) == case["bytes"]
        assert list(o.unpack_int4(b)[0]) == case["codes"]


def pin_hand_gemm(o):
    g = _golden()
    acts = {c["name"]: c for c in g["activation_cases"]}
    wts = {c["name"]: c for c in g["weight_cases"]}
    for case in g["gemm_cases"]:
        a, w = acts[case["act_case"]], wts[case["weight_case"]]
        qa, sa = o.quantize_groups(_pad32(a["x"]), a["c"], a["bits"])
        qw, sw = o.quantize_weights(_pad32(w["w"]))
        y = o.group_gemm(qa, sa, qw, sw)
        assert int((qa.astype(np.int64) @ qw.astype(np.int64).T)[0, 0]) == case["acc"]
        assert y[0, 0] == case["y"]


def _exact_rtn(x: np.float32, s: np.float32, qmax: int) -> int:
    """Nearest level (ties to even) to fl32(x/s), decided in exact rational arithmetic.

    fl32(x/s) is formed as the float32 nearest to the exact quotient, found by
    enumerating neighbouring float32 values; the level choice uses Fractions.
    """
    if s == 0:
        return 0
    exact = Fraction(float(x)) / Fraction(float(s))
    # candidate float32 values around the double approximation
    approx = np.float32(float(exact))
    cands = [approx, np.nextafter(approx, np.float32(np.inf)),
             np.nextafter(approx, np.float32(-np.inf))]
    best = None
    for cnd in cands:
        d = abs(Fraction(float(cnd)) - exact)
        key = (d, int(np.float32(cnd).view(np.uint32)) & 1)  # tie -> even mantissa
        if best is None or key < best[0]:
            best = (key, cnd)
    r = Fraction(float(best[1]))
    fl = r.numerator // r.denominator
    frac = r - fl
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return max(-qmax, min(qmax, fl))


def pin_rtn_bruteforce(o):
    rng = np.random.default_rng(11)
    for bits in (4, 8):
        qmax = (1 << (bits - 1)) - 1
        for c in (1.0, 0.8125, 0.7, 1.3):
            x = (rng.standard_normal((3, 64)) * 3).astype(np.float32)
            x[0, 5] = 0.0
            x[1, :32] = 0.0  # one all-zero group
            q, s = o.quantize_groups(x, c, bits)
            for m in range(x.shape[0]):
                for g in range(2):
                    blk = x[m, 32 * g:32 * g + 32]
                    amax = Fraction(float(np.abs(blk).max()))
                    # s = fl32(fl32(c*amax)/qmax): check it lies within float32
                    # rounding of the exact value c*amax/qmax
                    exact_s = Fraction(float(np.float32(c))) * amax / qmax
                    sv = s[m, g]
                    if exact_s == 0:
                        assert sv == 0
                    else:
                        assert abs(Fraction(float(sv)) - exact_s) <= exact_s * Fraction(1, 2 ** 22)
                    for k in range(32):
                        assert q[m, 32 * g + k] == _exact_rtn(blk[k], sv, qmax)


def pin_invariants(o):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((8, 256)) * 2).astype(np.float32)
    x[:, 7] *= 20
    for bits in (4, 8):
        qmax = (1 << (bits - 1)) - 1
        # c = 1: |q| <= qmax, absmax maps to +-qmax, reconstruction within s/2
        q, s = o.quantize_groups(x, 1.0, bits)
        assert np.abs(q).max() <= qmax
        xg = x.reshape(8, -1, 32)
        qg = q.reshape(8, -1, 32).astype(np.float64)
        idx = np.abs(xg).argmax(axis=2)
        top = np.take_along_axis(qg, idx[..., None], 2)[..., 0]
        assert np.all(np.abs(top) == qmax)
        err = np.abs(xg.astype(np.float64) - s[..., None].astype(np.float64) * qg)
        assert np.all(err <= s[..., None].astype(np.float64) * (0.5 + 1e-6))
        # c < 1: entries beyond the clip saturate, others reconstruct within s/2
        q2, s2 = o.quantize_groups(x, 0.7, bits)
        q2g = q2.reshape(8, -1, 32).astype(np.float64)
        r = xg.astype(np.float64) / s2[..., None]
        inside = np.abs(r) <= qmax
        err2 = np.abs(xg - s2[..., None] * q2g)
        assert np.all(err2[inside] <= (s2[..., None] * (0.5 + 1e-6) * np.ones_like(err2))[inside])
        assert np.all(np.abs(q2g[~inside]) == qmax)
        # odd symmetry Q(-x) = -Q(x)
        qn, sn = o.quantize_groups(-x, 0.9, bits)
        qp, sp = o.quantize_groups(x, 0.9, bits)
        assert np.array_equal(qn, -qp) and np.array_equal(sn, sp)
        # power-of-two scaling: codes unchanged, scales scale exactly
        q4, s4 = o.quantize_groups(x * np.float32(4.0), 0.9, bits)
        assert np.array_equal(q4, qp) and np.array_equal(s4, sp * np.float32(4.0))


def pin_kron(o):
    rng = np.random.default_rng(3)
    # dense Kronecker product for K = 256
    P1 = synth.orthogonal(16, 0, 0, 1)
    P2 = synth.orthogonal(16, 0, 0, 2)
    x = rng.standard_normal((5, 256)).astype(np.float32)
    assert np.array_equal(o.kron_rotate(x, P1, P2), o.kron_rotate_dense(x, P1, P2)) or \
        np.max(np.abs(o.kron_rotate(x, P1, P2) - o.kron_rotate_dense(x, P1, P2))) <= 1e-6
    # element-by-element brute force of x (P1 kron P2) on K = 12 (a = 3, b = 4)
    A = rng.standard_normal((3, 3)).astype(np.float32)
    B = rng.standard_normal((4, 4)).astype(np.float32)
    xs = rng.standard_normal((2, 12)).astype(np.float32)
    want = np.zeros((2, 12))
    for m in range(2):
        for col in range(12):
            i, j = divmod(col, 4)
            tot = 0.0
            for row in range(12):
                p, q = divmod(row, 4)
                tot += float(xs[m, row]) * float(A[p, i]) * float(B[q, j])
            want[m, col] = tot
    got = o.kron_rotate(xs, A, B)
    assert np.max(np.abs(got - want)) <= 1e-5
    # rounded once: each element is the float32 nearest to the exact rational
    # sum (float64 arithmetic is 2^-29 closer than float32's half-ulp, so a
    # double rounding could only differ within 2^-29 ulp of a tie; none is)
    for m in range(2):
        for col in range(12):
            i, j = divmod(col, 4)
            exact = sum(Fraction(float(xs[m, row])) * Fraction(float(A[row // 4, i]))
                        * Fraction(float(B[row % 4, j])) for row in range(12))
            below = np.float32(float(exact))
            cands = [below, np.nextafter(below, np.float32(np.inf)),
                     np.nextafter(below, np.float32(-np.inf))]
            nearest = min(cands, key=lambda c: abs(Fraction(float(c)) - exact))
            assert got[m, col] == nearest, (m, col)
    # P1 = swap, P2 = I maps [x0,x1,x2,x3] -> [x2,x3,x0,x1]
    v = np.array([[1.0, 2.0, 3.0, 4.0]], np.float32)
    swap = np.array([[0, 1], [1, 0]], np.float32)
    eye = np.eye(2, dtype=np.float32)
    assert list(o.kron_rotate(v, swap, eye)[0]) == [3.0, 4.0, 1.0, 2.0]
    # P1 = I, P2 = diag(1, -1) maps it to [x0, -x1, x2, -x3]
    d = np.diag([1.0, -1.0]).astype(np.float32)
    assert list(o.kron_rotate(v, eye, d)[0]) == [1.0, -2.0, 3.0, -4.0]
    # identity factors: exact identity
    xi = rng.standard_normal((3, 64)).astype(np.float32)
    assert np.array_equal(o.kron_rotate(xi, np.eye(8, dtype=np.float32),
                                         np.eye(8, dtype=np.float32)), xi)


def pin_fold_invariance(o):
    """P orthogonal => x W^T = (x P)(W P)^T; general invertible P uses P^{-T} on the weights."""
    rng = np.random.default_rng(4)
    # float64 orthogonal factors (the float32-stored ones are orthogonal to ~1e-7 only)
    P1 = np.linalg.qr(rng.standard_normal((16, 16)))[0]
    P2 = np.linalg.qr(rng.standard_normal((16, 16)))[0]
    x = rng.standard_normal((4, 256))
    W = rng.standard_normal((6, 256))
    P = np.kron(P1, P2)
    assert np.max(np.abs(P @ P.T - np.eye(256))) < 1e-12
    Pf = np.kron(synth.orthogonal(16, 0, 1, 1).astype(np.float64),
                 synth.orthogonal(16, 0, 1, 2).astype(np.float64))
    assert np.max(np.abs(Pf @ Pf.T - np.eye(256))) < 1e-6
    lhs = x @ W.T
    rhs = (x @ P) @ (W @ P).T
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(lhs)) * 256
    # non-orthogonal invertible factors: fold with the inverse-transpose
    A = rng.standard_normal((4, 4)) + 4 * np.eye(4)
    B = rng.standard_normal((8, 8)) + 4 * np.eye(8)
    xs = rng.standard_normal((3, 32))
    Ws = rng.standard_normal((5, 32))
    Wf = o.fold_weights(Ws.astype(np.float32), o.inverse_transpose(A), o.inverse_transpose(B))
    xr = (xs @ np.kron(A, B))
    assert np.max(np.abs(xr @ Wf.astype(np.float64).T - xs @ Ws.T)) < 1e-4


def pin_gemm_bruteforce(o):
    rng = np.random.default_rng(8)
    for K in (32, 64):
        M, N = 3, 4
        qa = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
        qw = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
        sa = rng.uniform(0.01, 1, size=(M, K // 32)).astype(np.float32)
        sw = rng.uniform(0.01, 1, size=(N, K // 32)).astype(np.float32)
        y = o.group_gemm(qa, sa, qw, sw)
        for m in range(M):
            for n in range(N):
                tot = Fraction(0)
                for g in range(K // 32):
                    acc = sum(int(qa[m, k]) * int(qw[n, k]) for k in range(32 * g, 32 * g + 32))
                    tot += Fraction(float(sa[m, g])) * Fraction(float(sw[n, g])) * acc
                assert abs(Fraction(float(y[m, n])) - tot) <= abs(tot) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 60)


def pin_special_cases(o):
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    # group = K reduces to one scale per token (per-token RTN arm)
    q, s = o.quantize_groups(x, 1.0, 4, group=128)
    assert s.shape == (4, 1)
    assert np.array_equal(s[:, 0], np.abs(x).max(1) / np.float32(7))
    # P = I: the rotate+quantize path is plain group RTN
    eye = np.eye(8, dtype=np.float32)
    q1, s1 = o.quantize_activation(x, np.eye(16, dtype=np.float32), eye, 0.9, 4)
    q2, s2 = o.quantize_groups(x, 0.9, 4)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)
    # unit scales: the GEMM reduces to an integer matmul
    qa = rng.integers(-7, 8, size=(5, 64)).astype(np.int8)
    qw = rng.integers(-7, 8, size=(3, 64)).astype(np.int8)
    ones_a = np.ones((5, 2), np.float32)
    ones_w = np.ones((3, 2), np.float32)
    assert np.array_equal(o.group_gemm(qa, ones_a, qw, ones_w),
                          (qa.astype(np.int64) @ qw.astype(np.int64).T).astype(np.float64))


def pin_loop_clip_index(o):
    """Loop t quantizes with its own clip c_t = las[t] (paper_specification.yaml:
    las, c_{t,l} per module and loop): a hand-worked case with four distinct
    clips, identity transforms and an exactly quantizable weight, through both
    the single-step call and the open- and chain-mode drivers."""
    (case,) = _golden()["loop_cases"]
    K, n = case["K"], len(case["x"])
    T = len(case["las"])
    W = np.float32(0.875) * np.eye(K, dtype=np.float32)
    layer = o.OracleLayer(W, np.eye(case["a"], dtype=np.float32),
                          np.eye(case["b"], dtype=np.float32),
                          np.asarray(case["las"], np.float32), 4)
    x = _pad32(case["x"])
    ys = o.loop_stack_open([[x] for _ in range(T)], [layer], T)
    for t in range(T):
        want = np.zeros((1, K))
        want[0, :n] = case["y"][t]
        assert np.array_equal(ys[t][0], want), f"loop {t}"
        assert np.array_equal(o.loop_linear(x, layer, t), want), f"loop {t}"
    # chain mode feeds y back; loop 1 must still clip with c_1 (its input is
    # loop 0's output, 0.875 * the codes of case w4a4_c1: absmax 6.125)
    ch = o.loop_stack_chain(x, [layer], 2)
    y0 = ch[0][0].astype(np.float32)
    s1 = np.float32(np.float32(case["las"][1]) * np.float32(6.125)) / np.float32(7)
    assert s1 == np.float32(0.4375)
    q1 = np.clip(np.rint(y0 / s1), -7, 7)  # y0 / s1 = 2 * the t = 0 codes, no ties
    assert np.array_equal(ch[1][0], 0.875 * np.float64(s1) * q1.astype(np.float64))


ALL_PINS = [pin_hand_activation, pin_hand_weight, pin_hand_packing, pin_hand_gemm,
            pin_rtn_bruteforce, pin_invariants, pin_kron, pin_fold_invariance,
            pin_gemm_bruteforce, pin_special_cases, pin_loop_clip_index]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(O)


def test_loop_driver_reductions():
    """T = 1 reduces the loop to one quantized linear; chain mode feeds y back."""
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    layer = O.OracleLayer(mp.W, mp.P1, mp.P2, mp.las, 4)
    x0 = synth.loop_input(wl, mp.lin, 0)
    ys = O.loop_stack_open([[x0]], [layer], 1)
    assert np.array_equal(ys[0][0], layer.forward(x0, 0))
    ch = O.loop_stack_chain(x0, [layer], 3)
    assert np.array_equal(ch[1][0], layer.forward(ch[0][0].astype(np.float32), 1))
    with pytest.raises(ValueError):
        layer.forward(x0, 4)
    # the quantized layer approximates the unquantized folded product
    y_ref = x0.astype(np.float64) @ mp.W.astype(np.float64).T
    y_q = layer.forward(x0, 0)
    rel = np.linalg.norm(y_q - y_ref) / np.linalg.norm(y_ref)
    assert rel < 0.2


def test_slt_schedule_reductions():
    """SLT serving: with every loop mapped to the shared layer it is the plain
    open / chain schedule; a loop-dependent layer at loop t gives, at that
    step, exactly the single-layer result of that layer, and a loop-dependent
    transform P_t with the weight folded by the same P_t still approximates
    x W^T (Section 2, Eqs. (2)-(3): folding keeps the product up to
    quantization), while a weight folded by another loop's transform does not."""
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    shared = O.OracleLayer(mp.W, mp.P1, mp.P2, mp.las, 4)
    xs = [[synth.loop_input(wl, mp.lin, t)] for t in range(3)]
    assert all(np.array_equal(a[0], b[0]) for a, b in
               zip(O.loop_stack_slt_open(xs, [[shared]] * 3, 3), O.loop_stack_open(xs, [shared], 3)))
    ch_a = O.loop_stack_slt_chain(xs[0][0], [[shared]] * 3, 3)
    ch_b = O.loop_stack_chain(xs[0][0], [shared], 3)
    assert all(np.array_equal(a[0], b[0]) for a, b in zip(ch_a, ch_b))
    # loop 1 gets its own transform pair and the weight folded with it
    rng = np.random.default_rng(5)
    P1t = np.linalg.qr(rng.standard_normal((16, 16)))[0].astype(np.float32)
    P2t = np.linalg.qr(rng.standard_normal((16, 16)))[0].astype(np.float32)
    own = O.OracleLayer(mp.W, P1t, P2t, mp.las, 4)
    ys = O.loop_stack_slt_open(xs, [[shared], [own], [shared]], 3)
    assert np.array_equal(ys[1][0], own.forward(xs[1][0], 1))
    assert np.array_equal(ys[0][0], shared.forward(xs[0][0], 0))
    y_ref = xs[1][0].astype(np.float64) @ mp.W.astype(np.float64).T
    rel = np.linalg.norm(ys[1][0] - y_ref) / np.linalg.norm(y_ref)
    assert rel < 0.2
    # mismatched pair: rotate with P_t but multiply the shared fold
    mixed = O.OracleLayer(mp.W, P1t, P2t, mp.las, 4, Q1=shared.Q1, Q2=shared.Q2)
    rel_bad = np.linalg.norm(mixed.forward(xs[1][0], 1) - y_ref) / np.linalg.norm(y_ref)
    assert rel_bad > 0.5


def test_cta_pins():
    """CTA (cta, Section 4.3, Eq. (7) as read: h' = a*h + b + eta*(h V) U^T):
    identity at initialization, the affine part alone when the gate is 0, the
    low-rank term against a brute-force sum in exact rationals, and a chained
    schedule whose transition is the identity equals plain chain mode."""
    rng = np.random.default_rng(3)
    M, d, r = 5, 64, 8
    h = rng.standard_normal((M, d)).astype(np.float32)
    U = (0.1 * rng.standard_normal((d, r))).astype(np.float32)
    V = (0.1 * rng.standard_normal((d, r))).astype(np.float32)
    a = (1 + 0.1 * rng.standard_normal(d)).astype(np.float32)
    b = (0.1 * rng.standard_normal(d)).astype(np.float32)
    one, zero = np.ones(d, np.float32), np.zeros(d, np.float32)
    assert np.array_equal(O.cta_apply(h, one, zero, 0.0, U, V), h)        # identity init
    aff = (a.astype(np.float64) * h.astype(np.float64) + b).astype(np.float32)
    assert np.array_equal(O.cta_apply(h, a, b, 0.0, U, V), aff)          # gate closed
    # low-rank term in exact arithmetic: sum_r (sum_k h_k V_kr) U_jr
    from fractions import Fraction
    eta = np.float32(0.37)
    got = O.cta_apply(h[:2, :16], one[:16], zero[:16], eta, U[:16], V[:16])
    for m in range(2):
        for j in range(16):
            p = [sum(Fraction(float(h[m, k])) * Fraction(float(V[k, q])) for k in range(16))
                 for q in range(r)]
            exact = Fraction(float(h[m, j])) + Fraction(float(eta)) * sum(
                p[q] * Fraction(float(U[j, q])) for q in range(r))
            # one float32 rounding of a value computed to float64 accuracy
            assert abs(float(got[m, j]) - float(exact)) <= 2 ** -23 * abs(float(exact)) + 1e-30
    # with identity transitions the CTA schedule is the plain chain schedule
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    layer = O.OracleLayer(mp.W, mp.P1, mp.P2, mp.las, 4)
    x0 = synth.loop_input(wl, mp.lin, 0)
    K = x0.shape[1]
    ones, zeros = np.ones(K, np.float32), np.zeros(K, np.float32)
    U0 = np.zeros((K, r), np.float32)
    a_c = [ones] * 3
    b_c = [zeros] * 3
    c1 = O.loop_stack_chain_cta(x0, [layer], 4, a_c, b_c, [0.0] * 3, U0, U0)
    c2 = O.loop_stack_chain(x0, [layer], 4)
    assert all(np.array_equal(p[0], q[0]) for p, q in zip(c1, c2))
    # a real transition changes the next loop's input and therefore its output
    c3 = O.loop_stack_chain_cta(x0, [layer], 2, [a.repeat(4)[:K]] * 1, [b.repeat(4)[:K]] * 1,
                                [0.5], np.tile(U, (4, 1)), np.tile(V, (4, 1)))
    assert np.array_equal(c3[0][0], c2[0][0]) and not np.array_equal(c3[1][0], c2[1][0])


def test_trajectory_hessian_pins():
    """H = sum_t X_t^T X_t: brute force over (t, m, i, j) in exact rationals on
    a tiny case, symmetry and positive semi-definiteness, T = 1 gives X^T X,
    doubling the inputs quadruples H, and the sum over steps is the Hessian of
    the concatenated steps."""
    from fractions import Fraction
    rng = np.random.default_rng(4)
    xs = [synth.round_bf16(rng.standard_normal((3, 4)).astype(np.float32)) for _ in range(2)]
    H = O.trajectory_hessian(xs)
    for i in range(4):
        for j in range(4):
            exact = sum(Fraction(float(x[m, i])) * Fraction(float(x[m, j]))
                        for x in xs for m in range(3))
            assert H[i, j] == float(exact)  # bf16 products and these sums are exact in f64
    big = [synth.round_bf16(rng.standard_normal((50, 32)).astype(np.float32)) for _ in range(3)]
    Hb = O.trajectory_hessian(big)
    assert np.array_equal(Hb, Hb.T)
    assert np.linalg.eigvalsh(Hb).min() > -1e-9 * np.abs(Hb).max()
    x0 = big[0].astype(np.float64)
    assert np.allclose(O.trajectory_hessian(big[:1]), x0.T @ x0, rtol=0, atol=1e-12)
    assert np.allclose(O.trajectory_hessian([2 * x for x in big]), 4 * Hb, rtol=1e-15, atol=0)
    assert np.allclose(O.trajectory_hessian([np.concatenate(big)]), Hb, rtol=1e-13, atol=1e-12)


# ----------------------------------------------------------------------------
# planted mistakes: a copy of the oracle with one plausible error must fail a pin
# ----------------------------------------------------------------------------
def _mutant(**over):
    ns = types.SimpleNamespace(**{k: getattr(O, k) for k in dir(O) if not k.startswith("__")})
    for k, v in over.items():
        setattr(ns, k, v)
    # rebind helpers that call each other through the namespace
    if "quantize_groups" in over and "quantize_weights" not in over:
        ns.quantize_weights = lambda Wt, group=32: ns.quantize_groups(Wt, 1.0, 4, group)
    if ("quantize_groups" in over or "kron_rotate" in over) and "quantize_activation" not in over:
        def qa(x, P1, P2, c, bits, group=32):
            xt = ns.kron_rotate(x, P1, P2) if P1 is not None else np.asarray(x, np.float32)
            return ns.quantize_groups(xt, c, bits, group)
        ns.quantize_activation = qa
    if "kron_rotate" in over and "fold_weights" not in over:
        ns.fold_weights = lambda W, Q1, Q2: ns.kron_rotate(W, Q1, Q2)
    return ns


def _q_variant(rounding=np.rint, use_c=True, divide=True, clip=True, axis_k=True):
    def qg(xt, c, bits, group=32):
        xt = np.asarray(xt, np.float32)
        M, K = xt.shape
        qmax = (1 << (bits - 1)) - 1
        G = K // group
        xg = xt.reshape(M, G, group) if axis_k else xt.reshape(M, group, G).transpose(0, 2, 1)
        amax = np.abs(xg).max(axis=2)
        cc = np.float32(c) if use_c else np.float32(1.0)
        s = (cc * amax) / np.float32(qmax)
        with np.errstate(divide="ignore", invalid="ignore"):
            r = xg / s[:, :, None] if divide else xg * (np.float32(1) / s[:, :, None])
        q = rounding(r)
        if clip:
            q = np.clip(q, -qmax, qmax)
        q = np.where(s[:, :, None] == 0, 0, q)
        if not axis_k:
            q = q.transpose(0, 2, 1)
        return np.nan_to_num(q).astype(np.int8).reshape(M, K), s
    return qg


def _runs_all(o):
    for pin in ALL_PINS:
        pin(o)


def _gemm_fold_f32(qa, sa, qw, sw, group=32):
    """The group fold y += (s_a s_w) acc carried in float32 instead of float64."""
    qa = np.asarray(qa).astype(np.float32)
    qw = np.asarray(qw).astype(np.float32)
    G = qa.shape[1] // group
    y = np.zeros((qa.shape[0], qw.shape[0]), np.float32)
    for g in range(G):
        acc = qa[:, g * group:(g + 1) * group] @ qw[:, g * group:(g + 1) * group].T
        y += (np.asarray(sa, np.float32)[:, g][:, None] * np.asarray(sw, np.float32)[:, g][None, :]) * acc
    return y.astype(np.float64)


class _LayerFirstClip(O.OracleLayer):
    """Planted mistake: every loop quantizes with the clip of loop 0."""

    def forward(self, x, t):
        qa, sa = O.quantize_activation(x, self.P1, self.P2, float(self.las[0]), self.a_bits)
        return O.group_gemm(qa, sa, self.qw, self.sw)


class _LayerNextClip(O.OracleLayer):
    """Planted mistake: loop t quantizes with the clip of loop t + 1 (wrapping)."""

    def forward(self, x, t):
        c = float(self.las[(t + 1) % self.las.size])
        qa, sa = O.quantize_activation(x, self.P1, self.P2, c, self.a_bits)
        return O.group_gemm(qa, sa, self.qw, self.sw)


MUTANTS = {
    "ties_away_from_zero": dict(quantize_groups=_q_variant(
        rounding=lambda r: np.sign(r) * np.floor(np.abs(r) + 0.5))),
    "dropped_las_clip": dict(quantize_groups=_q_variant(use_c=False)),
    "no_clip": dict(quantize_groups=_q_variant(clip=False)),
    "groups_strided_not_contiguous": dict(quantize_groups=_q_variant(axis_k=False)),
    "P1_not_transposed": dict(kron_rotate=lambda x, P1, P2: np.einsum(
        "ip,mpq,qj->mij", np.asarray(P1, np.float64),
        np.asarray(x, np.float64).reshape(len(x), P1.shape[0], P2.shape[0]),
        np.asarray(P2, np.float64)).reshape(len(x), -1).astype(np.float32)),
    "factors_swapped": dict(kron_rotate=lambda x, P1, P2: O.kron_rotate(x, P2, P1)
                            if P1.shape == P2.shape else O.kron_rotate(x, P1, P2) * 0),
    "pack_nibbles_swapped": dict(pack_int4=lambda c: (
        (np.asarray(c, np.int64) & 0xF)[..., 1::2] |
        ((np.asarray(c, np.int64) & 0xF)[..., 0::2] << 4)).astype(np.uint8)),
    "gemm_drops_weight_scale": dict(group_gemm=lambda qa, sa, qw, sw, group=32:
                                    O.group_gemm(qa, sa, qw, np.ones_like(sw), group)),
    "gemm_groups_misaligned": dict(group_gemm=lambda qa, sa, qw, sw, group=32:
                                   O.group_gemm(qa, sa[:, ::-1], qw, sw, group)),
    "quotient_by_reciprocal_multiply": dict(quantize_groups=_q_variant(divide=False)),
    "rotation_accumulated_in_float32": dict(kron_rotate=lambda x, P1, P2: np.einsum(
        "pi,mpq,qj->mij", np.asarray(P1, np.float32),
        np.asarray(x, np.float32).reshape(len(x), P1.shape[0], P2.shape[0]),
        np.asarray(P2, np.float32)).reshape(len(x), -1).astype(np.float32)),
    "gemm_fold_in_float32": dict(group_gemm=_gemm_fold_f32),
    "loop_uses_first_clip": dict(OracleLayer=_LayerFirstClip),
    "loop_uses_next_loop_clip": dict(OracleLayer=_LayerNextClip),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name):
    o = _mutant(**MUTANTS[name])
    with pytest.raises(AssertionError):
        _runs_all(o)
