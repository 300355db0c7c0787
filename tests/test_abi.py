"""Host-side checks of the C ABI (no GPU needed): the library builds, loads and
exports every entry point include/lq.h declares, and argument validation
rejects bad calls before anything is enqueued."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_ptq_looped_b200 import build as B
from bit_ptq_looped_b200 import lq

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "lq.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return lq.lib()


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for want in ("lq_quantize_act", "lq_pack_weights", "lq_loop_linear", "lq_loop_stack"):
        assert want in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert name in lq.SIGNATURES, f"binding lacks {name}"


def test_version(L):
    assert L.lq_version() == 100


def _err(L):
    return L.lq_last_error().decode()


def test_quantize_rejects_bad_arguments_before_launch(L):
    fake = 1 << 20  # never dereferenced: every call below fails its checks first
    # K not a multiple of 32
    st = L.lq_quantize_act(fake, lq.LQ_F32, 4, 48, None, 0, None, 0, 1.0, 4, 32, fake, None,
                           fake, None)
    assert st == lq.LQ_ERR_SHAPE and "multiple of 32" in _err(L)
    # unsupported bits / group
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, None, 0, None, 0, 1.0, 3, 32, fake, None,
                             fake, None) == lq.LQ_ERR_UNSUPPORTED
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, None, 0, None, 0, 1.0, 4, 64, fake, None,
                             fake, None) == lq.LQ_ERR_UNSUPPORTED
    # non-positive LAS clip
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, None, 0, None, 0, 0.0, 4, 32, fake, None,
                             fake, None) == lq.LQ_ERR_ARG
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, None, 0, None, 0, -1.0, 4, 32, fake, None,
                             fake, None) == lq.LQ_ERR_ARG
    # Kronecker sizes that do not multiply to K
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, fake, 4, fake, 8, 1.0, 4, 32, fake, None,
                             fake, None) == lq.LQ_ERR_SHAPE
    # only one factor
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, fake, 8, None, 0, 1.0, 4, 32, fake, None,
                             fake, None) == lq.LQ_ERR_ARG
    # factor sizes not multiples of 16 (a) and 8 (b)
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 96, fake, 6, fake, 16, 1.0, 4, 32, fake, None,
                             fake, None) == lq.LQ_ERR_UNSUPPORTED
    # packed output with 8-bit codes
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, None, 0, None, 0, 1.0, 8, 32, None, fake,
                             fake, None) == lq.LQ_ERR_UNSUPPORTED
    # misaligned pointer
    assert L.lq_quantize_act(fake + 4, lq.LQ_F32, 4, 64, None, 0, None, 0, 1.0, 4, 32, fake,
                             None, fake, None) == lq.LQ_ERR_ALIGN
    # unknown dtype, null outputs
    assert L.lq_quantize_act(fake, 7, 4, 64, None, 0, None, 0, 1.0, 4, 32, fake, None, fake,
                             None) == lq.LQ_ERR_UNSUPPORTED
    assert L.lq_quantize_act(fake, lq.LQ_F32, 4, 64, None, 0, None, 0, 1.0, 4, 32, None, None,
                             fake, None) == lq.LQ_ERR_ARG


def test_weight_entry_points_reject_bad_arguments(L):
    fake = 1 << 20
    h = ctypes.c_void_p()
    assert L.lq_pack_weights(fake, 16, 48, 4, 32, ctypes.byref(h), None) == lq.LQ_ERR_SHAPE
    assert L.lq_pack_weights(fake, 16, 64, 8, 32, ctypes.byref(h), None) == lq.LQ_ERR_UNSUPPORTED
    assert L.lq_pack_weights(fake, 0, 64, 4, 32, ctypes.byref(h), None) == lq.LQ_ERR_ARG
    assert L.lq_pack_weights(None, 16, 64, 4, 32, ctypes.byref(h), None) == lq.LQ_ERR_ARG
    assert L.lq_pack_weights(fake, 16, 64, 4, 32, None, None) == lq.LQ_ERR_ARG
    assert L.lq_quantize_weights(fake, 16, 64, 8, 32, fake, None, fake, None) == \
        lq.LQ_ERR_UNSUPPORTED
    # aliasing input and output
    assert L.lq_fold_weights(fake, 16, 128, fake, 16, fake, 8, fake, None) == lq.LQ_ERR_ARG
    assert L.lq_fold_weights(fake, 16, 64, fake, 4, fake, 8, fake + 16, None) == lq.LQ_ERR_SHAPE
    las = (ctypes.c_float * 2)(1.0, 0.5)
    assert L.lq_layer_create(None, fake, 4, fake, 4, las, 2, 4, ctypes.byref(h)) == lq.LQ_ERR_ARG


def test_loop_entry_points_reject_bad_arguments(L):
    fake = 1 << 20
    assert L.lq_loop_linear(fake, lq.LQ_F32, 4, None, 0, fake, fake, 1 << 20, None) == \
        lq.LQ_ERR_ARG
    assert L.lq_loop_stack(fake, lq.LQ_F32, 4, None, 1, 4, lq.LQ_OPEN, fake, fake, 1 << 20,
                           None) == lq.LQ_ERR_ARG
    assert L.lq_workspace_bytes(None, 1, 4) == -1
    assert L.lq_stack_workspace_bytes(None, 1, 4, 4) == -1
    assert L.lq_cta_stack_workspace_bytes(None, 1, 4) == -1
    assert L.lq_loop_stack_cta(fake, lq.LQ_F32, 4, None, 1, 4, None, fake, fake, 1 << 20,
                               None) == lq.LQ_ERR_ARG
    assert L.lq_loop_stack_slt(fake, lq.LQ_F32, 4, None, 1, 4, lq.LQ_OPEN, fake, fake, 1 << 20,
                               None) == lq.LQ_ERR_ARG
    assert L.lq_cta_apply(fake, 4, None, 0, fake, None) == lq.LQ_ERR_ARG
    out = ctypes.c_void_p()
    assert L.lq_cta_create(None, fake, 16, 8, fake, fake, None, 1, ctypes.byref(out)) == \
        lq.LQ_ERR_ARG


def test_selftests_reject_bad_arguments(L):
    """Both failure-path self-tests check their limit (and the grid wait its
    scratch) before any launch."""
    fake = 1 << 20
    for bad in (0, -1, 10**8):
        assert L.lq_selftest_bounded_wait(bad, None) == lq.LQ_ERR_ARG
        assert L.lq_selftest_grid_wait(bad, fake, None) == lq.LQ_ERR_ARG
    assert L.lq_selftest_grid_wait(1000, None, None) == lq.LQ_ERR_ARG
    assert L.lq_selftest_grid_wait(1000, fake + 2, None) == lq.LQ_ERR_ARG  # misaligned


def test_inverse_transpose_host_helper():
    rng = np.random.default_rng(0)
    for n in (1, 4, 16, 88):
        P = (rng.standard_normal((n, n)) + n * np.eye(n)).astype(np.float32)
        got = lq.lq_inverse_transpose(P).numpy()
        want = np.linalg.inv(P.astype(np.float64)).T
        assert np.max(np.abs(got - want)) <= 1e-6 * max(1.0, np.max(np.abs(want)))
    with pytest.raises(lq.LQError):
        lq.lq_inverse_transpose(np.zeros((3, 3), np.float32))


def test_size_functions(L):
    # lq_act_scale_bytes: one float32 step per row and group of 32
    for M, K in ((1, 32), (7, 2048), (2048, 5632)):
        assert L.lq_act_scale_bytes(M, K) == M * (K // 32) * 4
    # lq_hessian_workspace_bytes: the transposed bf16 inputs, K x (M*T rows, padded), 256-aligned
    assert L.lq_hessian_workspace_bytes(-1, 128, 1) == -1
    assert L.lq_hessian_workspace_bytes(4, 0, 1) == -1
    assert L.lq_hessian_workspace_bytes(4, 128, 0) == -1
    prev = 0
    for M, K, T in ((1, 128, 1), (5, 256, 4), (2048, 2048, 4), (2049, 2048, 4)):
        n = L.lq_hessian_workspace_bytes(M, K, T)
        assert n >= K * M * T * 2 and n % 256 == 0
        assert n < K * (M * T + 64) * 2 + 256  # padding below one 64-row block
        assert n >= prev
        prev = n


def test_hessian_entry_rejects_bad_arguments(L):
    fake = 1 << 20  # never dereferenced: every call below fails its checks first
    big = 1 << 40
    # inputs must be bf16
    assert L.lq_trajectory_hessian(fake, lq.LQ_F32, 4, 128, 2, fake, 0, fake, big, None) == \
        lq.LQ_ERR_UNSUPPORTED
    # shapes
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, -1, 128, 2, fake, 0, fake, big, None) == \
        lq.LQ_ERR_ARG
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, 4, 128, 0, fake, 0, fake, big, None) == \
        lq.LQ_ERR_ARG
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, 4, 100, 2, fake, 0, fake, big, None) == \
        lq.LQ_ERR_SHAPE
    # H: null, misaligned
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, 4, 128, 2, None, 0, fake, big, None) == \
        lq.LQ_ERR_ARG
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, 4, 128, 2, fake + 4, 0, fake, big, None) == \
        lq.LQ_ERR_ALIGN
    # no rows while accumulating: H stays as it is, nothing is enqueued
    assert L.lq_trajectory_hessian(None, lq.LQ_BF16, 0, 128, 2, fake, 1, None, 0, None) == lq.LQ_OK
    # X and workspace: null, misaligned, too small
    assert L.lq_trajectory_hessian(None, lq.LQ_BF16, 4, 128, 2, fake, 0, fake, big, None) == \
        lq.LQ_ERR_ARG
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, 4, 128, 2, fake, 0, fake + 16, big, None) == \
        lq.LQ_ERR_ALIGN
    assert L.lq_trajectory_hessian(fake, lq.LQ_BF16, 4, 128, 2, fake, 0, fake, 256, None) == \
        lq.LQ_ERR_WORKSPACE
