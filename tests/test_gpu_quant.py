"""GPU parity of the quantizers (lq_quantize_act, lq_quantize_weights,
lq_pack_weights, lq_fold_weights) against the CPU oracle."""
import numpy as np
import pytest
import torch

from bit_ptq_looped_b200 import lq, synth
from oracle import lq_oracle as O
from tests.parity import act_tensor, check_codes_near_tie, dev, host

pytestmark = pytest.mark.gpu


def _outlier_matrix(M, K, seed, frac=0.02, mult=20.0, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    ch = rng.choice(K, max(1, int(round(frac * K))), replace=False)
    x[:, ch] *= np.float32(mult)
    return x


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("x_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("c", [1.0, 0.7, 0.8374])
@pytest.mark.parametrize("shape", [(1, 32), (3, 64), (257, 256), (2048, 2048), (130, 5632)])
def test_quantize_only_bit_exact(bits, x_dtype, c, shape):
    M, K = shape
    x = _outlier_matrix(M, K, seed=M * 7 + K)
    if x_dtype == "bf16":
        x = synth.round_bf16(x)
    x[0, :32] = 0.0  # one all-zero group
    if M > 2:
        x[2, 32:64] = np.float32(3.5) * np.sign(x[2, 32:64])  # many exact ties
    q8, q4, s = lq.lq_quantize_act(act_tensor(x, x_dtype), None, None, c, bits,
                                   want_codes4=(bits == 4))
    torch.cuda.synchronize()
    q_or, s_or = O.quantize_groups(x, c, bits)
    np.testing.assert_array_equal(host(s), s_or)
    np.testing.assert_array_equal(host(q8), q_or)
    if bits == 4:
        np.testing.assert_array_equal(host(q4), O.pack_int4(q_or))


def test_quantize_only_edge_values():
    # powers of two, subnormal-range values and exact half-way ratios
    K = 64
    rows = [np.full(K, 7.0), np.linspace(-7, 7, K), np.full(K, 1e-39),
            np.concatenate([[2.0 ** -120], np.zeros(K - 1)]),
            np.arange(K) * 0.5 - 16, np.full(K, -3.0e37)]
    x = np.stack(rows).astype(np.float32)
    for bits in (4, 8):
        for c in (1.0, 0.75, 1.5):
            q8, _, s = lq.lq_quantize_act(dev(x), None, None, c, bits)
            torch.cuda.synchronize()
            q_or, s_or = O.quantize_groups(x, c, bits)
            np.testing.assert_array_equal(host(s), s_or)
            np.testing.assert_array_equal(host(q8), q_or)


def test_quantize_empty_input_is_a_noop():
    x = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    q8, _, s = lq.lq_quantize_act(x, None, None, 1.0, 4)
    torch.cuda.synchronize()
    assert q8.numel() == 0 and s.numel() == 0


WORKLOADS = [synth.TINY, synth.ATTN_PROJ, synth.MLP]


@pytest.mark.parametrize("wl", WORKLOADS, ids=lambda w: w.name)
@pytest.mark.parametrize("bits", [4, 8])
def test_fused_rotate_quantize(wl, bits):
    params = synth.module_params(wl)
    for l, (lin, mp) in enumerate(zip(wl.linears, params)):
        M = min(wl.M, 512) + (3 if wl.M > 64 else 0)  # several row tiles and a ragged tail
        for t in (0, wl.T - 1):
            x = synth.loop_input(wl, lin, t, rows=np.arange(M))
            c = float(mp.las[t])
            q8, q4, s = lq.lq_quantize_act(act_tensor(x, wl.x_dtype), dev(mp.P1), dev(mp.P2), c,
                                           bits, want_codes4=(bits == 4))
            torch.cuda.synchronize()
            xt64 = O.kron_rotate_f64(x, mp.P1, mp.P2)
            q_or, s_or = O.quantize_groups(xt64.astype(np.float32), c, bits)
            flips = check_codes_near_tie(host(q8), host(s), q_or, s_or, xt64)
            if bits == 4:
                np.testing.assert_array_equal(O.unpack_int4(host(q4)), host(q8))
            # the float64 rotation rounds like the oracle's: no differences expected here
            assert len(flips) == 0


def _orthogonal(n, seed):
    q, _ = np.linalg.qr(np.random.default_rng(seed).standard_normal((n, n)))
    return q.astype(np.float32)


@pytest.mark.parametrize("M", [1, 3, 16, 17])
@pytest.mark.parametrize("ab", [(32, 64), (64, 64), (16, 128), (64, 88), (16, 16)])
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_fused_rotate_quantize_few_rows(M, ab, x_dtype):
    """Up to 16 rows with b % 32 == 0 take the one-block-per-(row, 32 columns)
    kernel; other factor sizes and 17 rows take the row-tile kernel.  Both
    must give the oracle's codes (only near-tie differences allowed)."""
    a, b = ab
    K = a * b
    x = _outlier_matrix(M, K, seed=M * 131 + K)
    if x_dtype == "bf16":
        x = synth.round_bf16(x)
    P1, P2 = _orthogonal(a, a + 1), _orthogonal(b, b + 2)
    for bits in (4, 8):
        q8, q4, s = lq.lq_quantize_act(act_tensor(x, x_dtype), dev(P1), dev(P2), 0.83, bits,
                                       want_codes4=(bits == 4))
        torch.cuda.synchronize()
        xt64 = O.kron_rotate_f64(x, P1, P2)
        q_or, s_or = O.quantize_groups(xt64.astype(np.float32), 0.83, bits)
        flips = check_codes_near_tie(host(q8), host(s), q_or, s_or, xt64)
        assert len(flips) == 0
        if bits == 4:
            np.testing.assert_array_equal(O.unpack_int4(host(q4)), host(q8))


@pytest.mark.parametrize("ab,M", [((32, 64), 2368 + 37), ((64, 88), 592 + 5), ((16, 16), 9472 + 301),
                                  ((16, 128), 2368 * 2 + 1), ((64, 64), 1184 + 129)])
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_fused_rotate_quantize_many_rows(ab, M, x_dtype):
    """Enough rows for the warp-specialised kernel (one persistent block per
    SM, at least four row tiles per block; tiles of 16, 4 or 1 rows by factor
    size), with a ragged last tile and blocks holding one tile more than
    others: every code against the oracle (only near-tie differences)."""
    a, b = ab
    K = a * b
    x = _outlier_matrix(M, K, seed=M + K)
    if x_dtype == "bf16":
        x = synth.round_bf16(x)
    P1, P2 = _orthogonal(a, a + 5), _orthogonal(b, b + 6)
    xt64 = O.kron_rotate_f64(x, P1, P2)
    for bits in (4, 8):
        q8, q4, s = lq.lq_quantize_act(act_tensor(x, x_dtype), dev(P1), dev(P2), 0.91, bits,
                                       want_codes4=(bits == 4))
        torch.cuda.synchronize()
        q_or, s_or = O.quantize_groups(xt64.astype(np.float32), 0.91, bits)
        flips = check_codes_near_tie(host(q8), host(s), q_or, s_or, xt64)
        assert len(flips) == 0
        if bits == 4:
            np.testing.assert_array_equal(O.unpack_int4(host(q4)), host(q8))


@pytest.mark.parametrize("M", [3, 2368 + 37])
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_fused_rotate_quantize_extreme_exponents(M, x_dtype):
    """Inputs whose float->double widening takes every path: a row of
    subnormals only, rows mixing signed zeros and subnormals into normal
    values, a row near 1e30 and a row near 1e-30 (few rows: the per-row
    kernel; many: the warp-specialised one); every code against the oracle."""
    a, b = 32, 64
    K = a * b
    rng = np.random.default_rng(M + 7)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0] = (rng.standard_normal(K) * 1e-39).astype(np.float32)  # subnormal
    x[1, ::3] = 0.0
    x[1, 1::3] = -0.0
    x[1, 2::7] = np.float32(3e-41)
    x[2] *= np.float32(1e30)
    if M > 3:
        x[3] *= np.float32(1e-30)
        x[4:, 5::11] = -0.0
        x[4:, 9::13] = np.float32(-2e-40)
    if x_dtype == "bf16":
        x = synth.round_bf16(x)
    assert np.any((x != 0) & (np.abs(x) < np.finfo(np.float32).tiny))
    P1, P2 = _orthogonal(a, 41), _orthogonal(b, 42)
    xt64 = O.kron_rotate_f64(x, P1, P2)
    for bits in (4, 8):
        q8, _, s = lq.lq_quantize_act(act_tensor(x, x_dtype), dev(P1), dev(P2), 0.85, bits)
        torch.cuda.synchronize()
        q_or, s_or = O.quantize_groups(xt64.astype(np.float32), 0.85, bits)
        flips = check_codes_near_tie(host(q8), host(s), q_or, s_or, xt64)
        assert len(flips) == 0


def test_fused_rotation_identity_factors_reduce_to_plain_rtn():
    M, K = 100, 2048
    x = _outlier_matrix(M, K, seed=3)
    eye1, eye2 = np.eye(32, dtype=np.float32), np.eye(64, dtype=np.float32)
    q8, _, s = lq.lq_quantize_act(dev(x), dev(eye1), dev(eye2), 0.9, 4)
    torch.cuda.synchronize()
    q_or, s_or = O.quantize_groups(x, 0.9, 4)
    np.testing.assert_array_equal(host(s), s_or)
    np.testing.assert_array_equal(host(q8), q_or)


def test_weight_quantize_and_pack_bit_exact():
    wl = synth.MLP
    for mp in synth.module_params(wl):
        W = mp.W
        Wt = O.fold_weights(W, O.inverse_transpose(mp.P1), O.inverse_transpose(mp.P2))
        q8, q4, s = lq.lq_quantize_weights(dev(Wt))
        torch.cuda.synchronize()
        q_or, s_or = O.quantize_weights(Wt)
        np.testing.assert_array_equal(host(s), s_or)
        np.testing.assert_array_equal(host(q8), q_or)
        np.testing.assert_array_equal(host(q4), O.pack_int4(q_or))
        wq = lq.lq_pack_weights(dev(Wt))
        c4, sc = lq.wq_tensors(wq)
        np.testing.assert_array_equal(host(c4), O.pack_int4(q_or))
        np.testing.assert_array_equal(host(sc), s_or)
        info = wq.info()
        assert info["N"] == W.shape[0] and info["K"] == W.shape[1]
        wq.free()


@pytest.mark.parametrize("ab", [(16, 16), (32, 64), (64, 88)])
def test_fold_weights(ab):
    a, b = ab
    rng = np.random.default_rng(a * b)
    N = 300
    W = (rng.standard_normal((N, a * b)) * 0.02).astype(np.float32)
    P1 = synth.orthogonal(a, 1, 0, 1)
    P2 = synth.orthogonal(b, 1, 0, 2)
    Q1 = O.inverse_transpose(P1).astype(np.float32)
    Q2 = O.inverse_transpose(P2).astype(np.float32)
    got = host(lq.lq_fold_weights(dev(W), dev(Q1), dev(Q2)))
    torch.cuda.synchronize()
    want64 = O.kron_rotate_f64(W, Q1, Q2)
    want = want64.astype(np.float32)
    # float64 sums in a different order round to the same float32 except
    # within float64 rounding of a float32 rounding boundary
    ulp = np.spacing(np.abs(want))
    assert np.all(np.abs(got - want) <= ulp)
    assert (got != want).mean() < 1e-4
    # and W~ stays an exact-arithmetic fold: x W^T = (x P)(W~)^T up to float rounding
    x = rng.standard_normal((4, a * b))
    lhs = x @ W.astype(np.float64).T
    rhs = (x @ np.kron(P1.astype(np.float64), P2.astype(np.float64))) @ got.astype(np.float64).T
    assert np.max(np.abs(lhs - rhs)) <= 1e-5 * np.max(np.abs(lhs))


def test_hand_examples_through_the_kernels():
    """The hand-derived cases of tests/golden/qa_hand_examples.json (worked out
    from Section 2 Eq. (4) of the LoopQ specification under the readings stated
    there) through the CUDA quantizer and weight packer, bit for bit: steps,
    codes (the exact ties included, one of which separates a true division from
    a reciprocal multiply) and packed bytes."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "qa_hand_examples.json")) as f:
        gold = json.load(f)
    for case in gold["activation_cases"]:
        x = np.zeros((1, 32), np.float32)
        x[0, :len(case["x"])] = case["x"]
        q8, q4, s = lq.lq_quantize_act(dev(x), None, None, case["c"], case["bits"],
                                       want_codes4=case["bits"] == 4)
        torch.cuda.synchronize()
        n = len(case["codes"])
        if "scale" in case:
            want_s = np.float32(case["scale"])
        else:  # s = fl32(fl32(c * absmax) / q_max), as the case's note works it out
            qmax = 7 if case["bits"] == 4 else 127
            want_s = np.float32(np.float32(case["c"]) * np.float32(np.abs(case["x"]).max())) \
                / np.float32(qmax)
        assert host(s)[0, 0] == want_s, case["name"]
        assert list(host(q8)[0, :n]) == case["codes"], case["name"]
        assert not host(q8)[0, n:].any(), case["name"]
        if case["bits"] == 4:
            assert np.array_equal(host(q4)[0], O.pack_int4(host(q8))[0]), case["name"]
    for case in gold["weight_cases"]:
        w = np.zeros((1, 32), np.float32)
        w[0, :len(case["w"])] = case["w"]
        c4, sc = lq.wq_tensors(lq.lq_pack_weights(dev(w)))
        torch.cuda.synchronize()
        assert host(sc)[0, 0] == np.float32(case["scale"])
        codes = O.unpack_int4(host(c4))[0]
        assert list(codes[:len(case["codes"])]) == case["codes"]
        assert not codes[len(case["codes"]):].any()
    for case in gold["packing_cases"]:
        # weights equal to the codes themselves: step 1 when the absmax is 7
        w = np.zeros((1, 32), np.float32)
        w[0, :len(case["codes"])] = case["codes"]
        c4, _ = lq.wq_tensors(lq.lq_pack_weights(dev(w)))
        torch.cuda.synchronize()
        assert list(host(c4)[0, :len(case["bytes"])]) == case["bytes"]
