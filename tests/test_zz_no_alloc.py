"""lq_loop_linear_noalloc: the entry point for callers that cannot allocate
device memory (an enqueue hook that only receives its input and output
buffers, a serving loop that may not allocate after start-up).  It must give
the same results as lq_loop_linear, which takes a caller workspace, and keep
doing so on back-to-back calls that reuse its fixed scratch.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

from bit_ptq_looped_b200 import lq, synth
from oracle import lq_oracle as O
from tests.parity import act_tensor, check_gemm, dev, host, linear_parity, weight_parity

pytestmark = pytest.mark.gpu


def _layer(wl, a_bits):
    (mp,) = synth.module_params(wl)
    ol = O.OracleLayer(mp.W, mp.P1, mp.P2, mp.las, a_bits)
    wq = lq.lq_pack_weights(lq.lq_fold_weights(dev(mp.W), dev(ol.Q1), dev(ol.Q2)))
    layer = lq.lq_layer_create(wq, dev(mp.P1), dev(mp.P2), mp.las, a_bits)
    c4, sc = lq.wq_tensors(wq)
    layer.w_flips = weight_parity(host(c4), host(sc), ol)
    return layer, wq, mp, ol


def _against_oracle(y_na, x, wl, layer, mp, ol, t, a_bits):
    """The no-allocation result against the float64 oracle, under the same
    near-tie rule as every other parity test."""
    xd = act_tensor(x, wl.x_dtype)
    q8, _, s = lq.lq_quantize_act(xd, dev(mp.P1), dev(mp.P2), float(mp.las[t]), a_bits)
    torch.cuda.synchronize()
    linear_parity(host(y_na), x, ol, t, host(q8), host(s), layer.w_flips)


@pytest.mark.parametrize("wl,M,a_bits", [(synth.ATTN_PROJ, 2048, 4), (synth.ATTN_PROJ, 512, 8),
                                         (synth.TINY, 64, 4),
                                         (synth.decode_workload(4, 2048, 8), 4, 8)],
                         ids=["attn-w4a4", "attn-w4a8", "tiny", "decode-m4"])
def test_noalloc_matches_workspace_entry_point(wl, M, a_bits):
    layer, wq, mp, ol = _layer(wl, a_bits)
    (lin,) = wl.linears
    # two calls in a row with different inputs and loops: the second call must
    # not see anything the first one left in the shared scratch
    for t in (0, wl.T - 1):
        x = synth.loop_input(wl, lin, t, rows=np.arange(M))
        xd = act_tensor(x, wl.x_dtype)
        y_ref = lq.lq_loop_linear(xd, layer, t)
        y_na = torch.full_like(y_ref, float("nan"))
        lq.lq_loop_linear_noalloc(xd, layer, t, y=y_na)
        torch.cuda.synchronize()
        check_gemm(host(y_na), host(y_ref).astype(np.float64), what=f"noalloc t={t}")
        _against_oracle(y_na, x, wl, layer, mp, ol, t, a_bits)
    layer.free()
    wq.free()


def test_noalloc_smaller_call_after_larger_one():
    """A call with many rows leaves codes and steps of all its rows in the
    shared scratch; a following call with fewer rows (another loop, so other
    clips) must read only what it wrote itself."""
    wl = synth.ATTN_PROJ
    layer, wq, mp, ol = _layer(wl, 4)
    (lin,) = wl.linears
    for t, M in ((0, 2048), (2, 200), (1, 64)):
        x = synth.loop_input(wl, lin, t, rows=np.arange(M))
        y_na = torch.full((M, lin.N), float("nan"), device="cuda")
        lq.lq_loop_linear_noalloc(act_tensor(x, wl.x_dtype), layer, t, y=y_na)
        torch.cuda.synchronize()
        _against_oracle(y_na, x, wl, layer, mp, ol, t, 4)
    layer.free()
    wq.free()


def test_noalloc_rejects_calls_beyond_its_scratch():
    layer, wq, _, _ = _layer(synth.ATTN_PROJ, 4)
    need_per_row = 2048 + 2048 // 32 * 4
    M = lq.LQ_NOALLOC_SCRATCH_BYTES // need_per_row + 8
    x = torch.zeros((M, 2048), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((M, 2048), dtype=torch.float32, device="cuda")
    with pytest.raises(lq.LQError) as e:
        lq.lq_loop_linear_noalloc(x, layer, 0, y=y)
    assert e.value.status == lq.LQ_ERR_WORKSPACE
    assert "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0  # nothing was enqueued
    layer.free()
    wq.free()
