"""GPU parity of cross-loop transition alignment (lq_cta_apply, lq_loop_stack_cta)
against the CPU oracle."""
import numpy as np
import pytest
import torch

from bit_ptq_looped_b200 import lq, synth
from oracle import lq_oracle as O
from tests.parity import check_gemm, dev, host

pytestmark = pytest.mark.gpu


def _adapter(d, r, n_trans, seed, scale=0.05):
    rng = np.random.default_rng(seed)
    U = (scale * rng.standard_normal((d, r))).astype(np.float32)
    V = (scale * rng.standard_normal((d, r))).astype(np.float32)
    a = (1 + 0.1 * rng.standard_normal((n_trans, d))).astype(np.float32)
    b = (0.1 * rng.standard_normal((n_trans, d))).astype(np.float32)
    eta = rng.uniform(0.1, 0.9, n_trans).astype(np.float32)
    return U, V, a, b, eta


def _ulp_diff(x, y):
    xi = x.view(np.int32).astype(np.int64)
    yi = y.view(np.int32).astype(np.int64)
    return np.abs(xi - yi)


@pytest.mark.parametrize("M,d,r", [(1, 256, 8), (5, 2048, 8), (1000, 2048, 3), (37, 5632, 8)])
def test_cta_apply_matches_oracle(M, d, r):
    U, V, a, b, eta = _adapter(d, r, 3, seed=M + d + r)
    h = np.random.default_rng(M).standard_normal((M, d)).astype(np.float32) * 3
    cta = lq.lq_cta_create(dev(U), dev(V), dev(a), dev(b), eta)
    for t in range(3):
        out = host(lq.lq_cta_apply(dev(h), cta, t))
        torch.cuda.synchronize()
        ref = O.cta_apply(h, a[t], b[t], float(eta[t]), U, V)
        # both round a float64 value once: only values on a float32 rounding
        # boundary can differ, by one unit in the last place
        du = _ulp_diff(out, ref)
        assert du.max() <= 1 and (du > 0).mean() <= 1e-4, (du.max(), (du > 0).mean())
    cta.free()


def test_cta_apply_in_place_and_identity():
    d, M = 2048, 64
    h = np.random.default_rng(1).standard_normal((M, d)).astype(np.float32)
    U, V, a, b, eta = _adapter(d, 8, 2, seed=2)
    ident = lq.lq_cta_create(dev(U), dev(V), dev(np.ones((2, d), np.float32)),
                             dev(np.zeros((2, d), np.float32)), np.zeros(2, np.float32))
    hd = dev(h)
    lq.lq_cta_apply(hd, ident, 1, out=hd)  # identity at initialization, in place
    torch.cuda.synchronize()
    assert np.array_equal(host(hd), h)
    cta = lq.lq_cta_create(dev(U), dev(V), dev(a), dev(b), eta)
    ref = host(lq.lq_cta_apply(dev(h), cta, 0))
    hd = dev(h)
    lq.lq_cta_apply(hd, cta, 0, out=hd)
    torch.cuda.synchronize()
    assert np.array_equal(host(hd), ref)
    with pytest.raises(lq.LQError) as e:
        lq.lq_cta_apply(hd, cta, 2)
    assert e.value.status == lq.LQ_ERR_SHAPE


def test_cta_create_rejects_width_not_multiple_of_32():
    U, V, a, b, eta = _adapter(48, 8, 1, seed=8)
    with pytest.raises(lq.LQError) as e:
        lq.lq_cta_create(dev(U), dev(V), dev(a), dev(b), eta)
    assert e.value.status == lq.LQ_ERR_SHAPE


def _tiny_layer():
    from tests.test_gpu_linear import make_layer
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    return wl, mp, make_layer(mp, 4)


def test_loop_stack_cta_tiny_matches_oracle():
    """Chain mode with the adapter at the 3 transitions of T = 4 loops."""
    wl, mp, (layer, ol) = _tiny_layer()
    (lin,) = wl.linears
    K = lin.K
    U, V, a, b, eta = _adapter(K, 8, wl.T - 1, seed=5)
    cta = lq.lq_cta_create(dev(U), dev(V), dev(a), dev(b), eta)
    x0 = synth.loop_input(wl, lin, 0)
    y = host(lq.lq_loop_stack_cta(dev(x0), [layer], wl.T, cta, M=wl.M))
    y2 = host(lq.lq_loop_stack_cta(dev(x0), [layer], wl.T, cta, M=wl.M))  # graph replay
    torch.cuda.synchronize()
    assert np.array_equal(y, y2)
    ys = O.loop_stack_chain_cta(x0, [ol], wl.T, a, b, eta, U, V)
    for t in range(wl.T):
        check_gemm(y[t * wl.M * lin.N:(t + 1) * wl.M * lin.N].reshape(wl.M, lin.N), ys[t][0],
                   what=f"cta chain t={t}")
    cta.free()


@pytest.mark.parametrize("M", [300, 2048])
def test_loop_stack_cta_two_pass_state_matches_oracle(M):
    """The adapted state the last transition of the chained schedule leaves in
    the workspace (right after the codes and steps) must equal the oracle's
    CTA of that loop's output (both round a float64 value once: at most one
    unit in the last place on at most 1e-4 of the values); d = 2048, a ragged
    last 8-row block at M = 300."""
    from tests.test_gpu_linear import make_layer
    wl = synth.ATTN_PROJ
    (mp,) = synth.module_params(wl)
    layer, _ = make_layer(mp, 4)
    d, T = 2048, 3
    U, V, a, b, eta = _adapter(d, 8, T - 1, seed=M)
    cta = lq.lq_cta_create(dev(U), dev(V), dev(a), dev(b), eta)
    x0 = dev(synth.loop_input(wl, wl.linears[0], 0, rows=np.arange(M)))
    nws = lq.lq_cta_stack_workspace_bytes([layer], M)
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    y = host(lq.lq_loop_stack_cta(x0, [layer], T, cta, M=M, ws=ws))
    torch.cuda.synchronize()
    off = -(-lq.lq_workspace_bytes([layer], M) // 256) * 256
    state = host(ws[off:off + M * d * 4].view(torch.float32)).reshape(M, d)
    y_last = y[(T - 2) * M * d:(T - 1) * M * d].reshape(M, d)
    ref = O.cta_apply(y_last, a[T - 2], b[T - 2], float(eta[T - 2]), U, V)
    du = _ulp_diff(state, ref)
    assert du.max() <= 1 and (du > 0).mean() <= 1e-4, (du.max(), (du > 0).mean())
    cta.free()


def test_loop_stack_cta_identity_is_plain_chain():
    wl, mp, (layer, ol) = _tiny_layer()
    (lin,) = wl.linears
    K = lin.K
    U = np.zeros((K, 8), np.float32)
    ident = lq.lq_cta_create(dev(U), dev(U), dev(np.ones((3, K), np.float32)),
                             dev(np.zeros((3, K), np.float32)), np.zeros(3, np.float32))
    x0 = synth.loop_input(wl, lin, 0)
    y1 = lq.lq_loop_stack_cta(dev(x0), [layer], wl.T, ident, M=wl.M)
    y2 = lq.lq_loop_stack(dev(x0), [layer], wl.T, lq.LQ_CHAIN, M=wl.M)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_loop_stack_cta_rejects_bad_calls():
    wl, mp, (layer, ol) = _tiny_layer()
    (lin,) = wl.linears
    U, V, a, b, eta = _adapter(lin.K, 8, 2, seed=6)
    cta = lq.lq_cta_create(dev(U), dev(V), dev(a), dev(b), eta)
    x0 = dev(synth.loop_input(wl, lin, 0))
    with pytest.raises(lq.LQError) as e:  # T = 4 needs 3 transitions
        lq.lq_loop_stack_cta(x0, [layer], 4, cta, M=wl.M)
    assert e.value.status == lq.LQ_ERR_SHAPE
    U2, V2, a2, b2, eta2 = _adapter(512, 8, 3, seed=7)
    wide = lq.lq_cta_create(dev(U2), dev(V2), dev(a2), dev(b2), eta2)
    with pytest.raises(lq.LQError) as e:  # width 512 != state width 256
        lq.lq_loop_stack_cta(x0, [layer], 4, wide, M=wl.M)
    assert e.value.status == lq.LQ_ERR_SHAPE
