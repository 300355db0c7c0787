"""GPU parity of the quantized looped linear (lq_loop_linear, lq_loop_stack):
tensor-core GEMM for prefill-sized M, weight-streaming GEMV for decode M."""
import copy

import numpy as np
import pytest
import torch

from bit_ptq_looped_b200 import lq, synth
from oracle import lq_oracle as O
from tests.parity import act_tensor, check_gemm, dev, host, linear_parity, weight_parity

pytestmark = pytest.mark.gpu


def make_layer(mp, a_bits, T=None):
    """Fold with the float32 P^{-T} factors and pack on the device; return
    (lq Layer, oracle layer), with the weight-code near-tie differences in
    ``layer.w_flips``."""
    las = mp.las if T is None else mp.las[:T]
    ol = O.OracleLayer(mp.W, mp.P1, mp.P2, las, a_bits)
    Wf = lq.lq_fold_weights(dev(mp.W), dev(ol.Q1), dev(ol.Q2))
    wq = lq.lq_pack_weights(Wf)
    layer = lq.lq_layer_create(wq, dev(mp.P1), dev(mp.P2), las, a_bits)
    c4, sc = lq.wq_tensors(wq)
    layer.w_flips = weight_parity(host(c4), host(sc), ol)
    return layer, ol


def _integer_problem(M, N, K, a_bits, seed):
    """Integer codes whose every group holds +-q_max: all steps are exactly 1."""
    rng = np.random.default_rng(seed)
    qmax = 7 if a_bits == 4 else 127
    x = rng.integers(-qmax, qmax + 1, size=(M, K)).astype(np.float32)
    w = rng.integers(-7, 8, size=(N, K)).astype(np.float32)
    x[:, ::32] = qmax
    w[:, 1::32] = -7
    return x, w


@pytest.mark.parametrize("a_bits", [4, 8])
@pytest.mark.parametrize("MNK", [(128, 128, 128), (256, 384, 512), (200, 144, 2048),
                                 (1000, 2048, 256), (33, 256, 128)])
def test_gemm_exact_on_integer_problems(a_bits, MNK):
    """With unit steps the library must return the exact integer product."""
    M, N, K = MNK
    a = 16
    b = K // a
    x, w = _integer_problem(M, N, K, a_bits, seed=M + N + K)
    wq = lq.lq_pack_weights(dev(w))
    eye_a, eye_b = torch.eye(a, device="cuda"), torch.eye(b, device="cuda")
    layer = lq.lq_layer_create(wq, eye_a, eye_b, [1.0], a_bits)
    y = host(lq.lq_loop_linear(dev(x), layer, 0))
    torch.cuda.synchronize()
    want = x.astype(np.int64) @ w.astype(np.int64).T
    np.testing.assert_array_equal(y, want.astype(np.float32))


@pytest.mark.parametrize("a_bits", [4, 8])
@pytest.mark.parametrize("wl", [synth.TINY, synth.ATTN_PROJ, synth.MLP], ids=lambda w: w.name)
def test_loop_linear_prefill(wl, a_bits):
    params = synth.module_params(wl)
    for lin, mp in zip(wl.linears, params):
        layer, ol = make_layer(mp, a_bits)
        M = wl.M if wl.M <= 2048 else 2048
        for t in range(wl.T):
            x = synth.loop_input(wl, lin, t, rows=np.arange(M))
            xd = act_tensor(x, wl.x_dtype)
            y = lq.lq_loop_linear(xd, layer, t)
            q8, _, s = lq.lq_quantize_act(xd, dev(mp.P1), dev(mp.P2), float(mp.las[t]), a_bits)
            torch.cuda.synchronize()
            linear_parity(host(y), x, ol, t, host(q8), host(s), layer.w_flips)


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("N", [2048, 5632])
@pytest.mark.parametrize("a_bits", [8, 4])
def test_loop_linear_decode(M, N, a_bits):
    wl = synth.decode_workload(M, N, a_bits)
    (mp,) = synth.module_params(wl)
    (lin,) = wl.linears
    layer, ol = make_layer(mp, a_bits)
    for t in range(wl.T):
        x = synth.loop_input(wl, lin, t)
        xd = act_tensor(x, wl.x_dtype)
        y = lq.lq_loop_linear(xd, layer, t)
        q8, _, s = lq.lq_quantize_act(xd, dev(mp.P1), dev(mp.P2), float(mp.las[t]), a_bits)
        torch.cuda.synchronize()
        linear_parity(host(y), x, ol, t, host(q8), host(s), layer.w_flips)


def _gemv_case(M, N, K, a, b, a_bits, t=0):
    """One decode-sized linear (M tokens, K = a * b, N weight rows) through the
    library against the oracle."""
    wl = synth.Workload(f"decode_M{M}_N{N}_K{K}", M=M, T=t + 1,
                        linears=(synth.Linear("dec", K, N, a, b, 0),), a_bits=a_bits,
                        outlier_frac=0.02, outlier_mult=20.0, x_dtype="bf16",
                        description="decode GEMV case")
    (mp,) = synth.module_params(wl)
    (lin,) = wl.linears
    layer, ol = make_layer(mp, a_bits)
    x = synth.loop_input(wl, lin, t)
    xd = act_tensor(x, wl.x_dtype)
    y = lq.lq_loop_linear(xd, layer, t)
    q8, _, s = lq.lq_quantize_act(xd, dev(mp.P1), dev(mp.P2), float(mp.las[t]), a_bits)
    torch.cuda.synchronize()
    linear_parity(host(y), x, ol, t, host(q8), host(s), layer.w_flips)


@pytest.mark.parametrize("M", [1, 4, 6, 9, 16])
def test_gemv_many_row_batches(M):
    """N = 3 * 5632 + 8 weight rows: more rows than one resident wave of warps
    holds, so every warp folds several batches (dp4a) or several row blocks
    through its stage ring (tensor-core path, 6, 9 and 16 tokens: one and two
    blocks of 8 tokens, partly empty), and the last rows are ragged."""
    _gemv_case(M, 3 * 5632 + 8, 2048, 32, 64, 8)


@pytest.mark.parametrize("M,a_bits", [(1, 8), (2, 8), (3, 4), (4, 8), (4, 4)])
def test_gemv_streaming_few_tokens(M, a_bits):
    """A launch of more than one wave of 16-row blocks (N = 148 x 256 + 8
    rows): 2 to 4 tokens take the tensor-core path with its stage ring, one
    token the dp4a path with two weight-row batches in flight per warp; the
    last rows are ragged."""
    _gemv_case(M, 148 * 256 + 8, 2048, 32, 64, a_bits)


@pytest.mark.parametrize("K,a,b", [(128, 16, 8), (384, 16, 24), (1152, 16, 72), (5632, 64, 88)])
@pytest.mark.parametrize("M", [5, 16])
def test_gemv_tensor_core_group_tails(K, a, b, M):
    """Group counts against the stages of 16 (up to 8 tokens) and 8 groups
    (9 to 16 tokens): G = 4 (fewer groups than a stage), 12 and 36 (a partial
    last stage), 176 (whole stages); N = 1000 rows (a ragged row block)."""
    _gemv_case(M, 1000, K, a, b, 8)


def test_gemv_tensor_core_large_k():
    """K = 7680 = 96 x 80 at 16 tokens, the largest Kronecker shape the
    rotation stages: the activation fragments (150 KB) and three stages per
    warp fill 210 KB of shared memory."""
    _gemv_case(16, 520, 7680, 96, 80, 4)


@pytest.mark.parametrize("M", [0, 1, 17, 129, 300])
def test_loop_linear_ragged_rows(M):
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    (lin,) = wl.linears
    layer, ol = make_layer(mp, 4)
    rng = np.random.default_rng(M)
    x = rng.standard_normal((M, lin.K)).astype(np.float32)
    y = lq.lq_loop_linear(dev(x), layer, 2)
    torch.cuda.synchronize()
    if M == 0:
        assert y.numel() == 0
        return
    q8, _, s = lq.lq_quantize_act(dev(x), dev(mp.P1), dev(mp.P2), float(mp.las[2]), 4)
    torch.cuda.synchronize()
    linear_parity(host(y), x, ol, 2, host(q8), host(s), layer.w_flips)


def test_resident_weights_are_four_bit():
    """The resident weight object holds only the packed 4-bit codes and their
    float32 steps: N*K/2 + N*(K/32)*4 bytes, 0.625 bytes per weight; the
    tensor-core path expands its 8-bit operand into the call's workspace."""
    wl = synth.MLP
    for mp in synth.module_params(wl):
        layer, _ = make_layer(mp, 4)
        info = layer.wq.info()
        N, K = info["N"], info["K"]
        assert info["device_bytes"] == N * K // 2 + N * (K // 32) * 4
        assert info["device_bytes"] / (N * K) <= 0.66
        M = 256  # tensor-core path: the workspace holds the operand of this layer
        assert lq.lq_workspace_bytes([layer], M) >= M * K + N * K


def test_loop_linear_rejects_bad_calls():
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    layer, _ = make_layer(mp, 4)
    x = torch.zeros((64, 256), device="cuda")
    with pytest.raises(lq.LQError) as e:
        lq.lq_loop_linear(x, layer, 4)
    assert e.value.status == lq.LQ_ERR_SHAPE
    with pytest.raises(lq.LQError) as e:
        lq.lq_loop_linear(x, layer, -1)
    assert e.value.status == lq.LQ_ERR_SHAPE
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(lq.LQError) as e:
        lq.lq_loop_linear(x, layer, 0, ws=ws)
    assert e.value.status == lq.LQ_ERR_WORKSPACE


def _stack_inputs(wl, M):
    xs = [[synth.loop_input(wl, lin, t, rows=np.arange(M)) for lin in wl.linears]
          for t in range(wl.T)]
    flat = np.concatenate([xs[t][l].ravel() for t in range(wl.T) for l in range(len(wl.linears))])
    return xs, flat


@pytest.mark.parametrize("wl,M", [(synth.TINY, 64), (synth.MLP, 2048), (synth.ATTN_PROJ, 2048)],
                         ids=["tiny", "mlp", "attn"])
def test_loop_stack_open(wl, M):
    """Open-mode stack with the default workspace, sized for all T loops: one
    rotate+quantize launch and one GEMM launch per linear for the 4 loops (the
    launch configuration the benchmark times for these workloads, at their full
    sizes: M = 2048; the MLP's down projection runs 8192 rows of K = 5632 per
    launch); every output of every loop against the oracle, and graph replays
    bit-identical."""
    params = synth.module_params(wl)
    built = [make_layer(mp, wl.a_bits) for mp in params]
    layers = [b[0] for b in built]
    xs, flat = _stack_inputs(wl, M)
    xd = act_tensor(flat, wl.x_dtype)
    y1 = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M)
    y2 = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M, y=torch.empty_like(y1))
    y3 = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M, y=y1)  # graph replay, same args
    torch.cuda.synchronize()
    y1h = host(y1)
    assert np.array_equal(y1h, host(y2)) and np.array_equal(y1h, host(y3))
    off = 0
    for t in range(wl.T):
        for l, (lin, mp) in enumerate(zip(wl.linears, params)):
            n = M * lin.N
            yg = y1h[off:off + n].reshape(M, lin.N)
            off += n
            xd_tl = act_tensor(xs[t][l], wl.x_dtype)
            q8, _, s = lq.lq_quantize_act(xd_tl, dev(mp.P1), dev(mp.P2), float(mp.las[t]),
                                          wl.a_bits)
            torch.cuda.synchronize()
            linear_parity(yg, xs[t][l], built[l][1], t, host(q8), host(s), built[l][0].w_flips)


@pytest.mark.parametrize("wl,M", [(synth.MLP, 256), (synth.TINY, 64), (synth.ATTN_PROJ, 200)],
                         ids=["mlp", "tiny", "attn_ragged"])
def test_loop_stack_open_batching_matches_per_loop(wl, M):
    """Open mode runs several loops of a layer per launch when the workspace
    holds them.  Each output row goes through the same per-row arithmetic, so
    every batch width (including a partial last batch, and M not a multiple of
    the 128-row GEMM tile) must reproduce the one-loop-per-launch schedule bit
    for bit."""
    params = synth.module_params(wl)
    layers = [make_layer(mp, wl.a_bits)[0] for mp in params]
    xs, flat = _stack_inputs(wl, M)
    xd = act_tensor(flat, wl.x_dtype)
    T = wl.T
    ref = lq.lq_loop_stack(xd, layers, T, lq.LQ_OPEN, M=M, ws=lq.workspace(layers, M))
    for nb in (2, 3, T):
        ws = lq.workspace(layers, M, T=nb)
        # room for the codes and steps of nb loops (beside one weight operand)
        kmax = max(lin.K for lin in wl.linears)
        assert ws.numel() >= lq.lq_workspace_bytes(layers, M) + (nb - 1) * M * kmax
        y = lq.lq_loop_stack(xd, layers, T, lq.LQ_OPEN, M=M, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(y, ref), f"batch of {nb} loops"


@pytest.mark.parametrize("M,a_bits", [(1, 8), (3, 4), (4, 4), (16, 8)])
def test_loop_stack_open_decode_branches(M, a_bits):
    """Decode-sized open mode: the loops of a layer form one unit while their
    rows fit the GEMV path (all 4 loops at 1, 3 and 4 tokens, one loop at 16).
    With the stack's workspace size every unit runs in one grouped quantize and
    one grouped GEMV launch; a workspace for one linear at T * M rows runs the
    units as two concurrent quantize->GEMV chains on internal streams (smaller
    loop batches), and a minimal workspace as one chain of one launch pair per
    loop.  Three linears of different widths (the last with a ragged N),
    T = 4: every output of all three schedules against the oracle, and the
    grouped schedule deterministic (bit-identical on a second call)."""
    lins = (synth.Linear("d0", 2048, 2048, 32, 64, 0), synth.Linear("d1", 2048, 5632, 32, 64, 0),
            synth.Linear("d2", 2048, 1000, 32, 64, 1))
    wl = synth.Workload(f"decode_stack_M{M}", M=M, T=4, linears=lins, a_bits=a_bits,
                        outlier_frac=0.02, outlier_mult=20.0, x_dtype="bf16",
                        description="decode stack of three linears")
    params = synth.module_params(wl)
    built = [make_layer(mp, a_bits) for mp in params]
    layers = [b[0] for b in built]
    xs, flat = _stack_inputs(wl, M)
    xd = act_tensor(flat, wl.x_dtype)
    ws_all = lq.workspace(layers, M, T=wl.T)
    ws_one = lq.workspace(layers, M)
    assert ws_all.numel() >= 2 * ws_one.numel()
    y = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M, ws=ws_all)
    y1 = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M, ws=ws_one)
    y2 = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M, ws=ws_all, y=torch.empty_like(y))
    # one linear at T * M rows: two chains of half-size loop batches (at 16
    # tokens this size, taken by the tensor-core path's operand, holds the
    # grouped schedule's regions)
    ws_seq = lq.workspace(layers, M * wl.T)
    ys = lq.lq_loop_stack(xd, layers, wl.T, lq.LQ_OPEN, M=M, ws=ws_seq)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    quant = {}
    for yy in (y, y1, ys):
        yh = host(yy)
        off = 0
        for t in range(wl.T):
            for l, (lin, mp) in enumerate(zip(wl.linears, params)):
                n = M * lin.N
                yg = yh[off:off + n].reshape(M, lin.N)
                off += n
                if (t, l) not in quant:
                    q8, _, s = lq.lq_quantize_act(act_tensor(xs[t][l], wl.x_dtype),
                                                  dev(mp.P1), dev(mp.P2), float(mp.las[t]),
                                                  a_bits)
                    torch.cuda.synchronize()
                    quant[(t, l)] = (host(q8), host(s))
                q8h, sh = quant[(t, l)]
                linear_parity(yg, xs[t][l], built[l][1], t, q8h, sh, built[l][0].w_flips)


@pytest.mark.parametrize("M,T,copies,a_bits,x_dtype", [
    (5, 4, 1, 8, "bf16"),    # loop batches of 3 and 1 (15 and 5 rows) in one launch
    (2, 4, 1, 4, "f32"),     # 8 rows: one token block
    (16, 4, 7, 8, "bf16"),   # 112 units of one loop: two rounds of 56
])
def test_loop_stack_open_decode_grouped(M, T, copies, a_bits, x_dtype):
    """Decode-sized open mode with the stack's own workspace size: every
    (layer, loop batch) unit of a round in one quantize launch and one GEMV
    launch (two launches per round, counted by the probe), each unit with its
    own rows (ragged loop batches share a launch), layers of different widths
    (factors 16x32 to 64x88) including a ragged N; every output of every loop
    against the oracle."""
    lins = (synth.Linear("g0", 512, 256, 16, 32, 0), synth.Linear("g1", 2048, 1000, 32, 64, 1),
            synth.Linear("g2", 1024, 96, 32, 32, 2), synth.Linear("g3", 5632, 200, 64, 88, 3))
    nl = len(lins)
    wl = synth.Workload(f"decode_grouped_M{M}", M=M, T=T, linears=lins, a_bits=a_bits,
                        outlier_frac=0.02, outlier_mult=20.0, x_dtype=x_dtype,
                        description="grouped decode stack")
    params = synth.module_params(wl)
    built = [make_layer(mp, a_bits) for mp in params]
    # the stack repeats the four linears `copies` times (same handles)
    L = nl * copies
    layers = [built[l % nl][0] for l in range(L)]
    xs = [[synth.loop_input(wl, lins[l % nl], t, rows=np.arange(M) + M * (l // nl))
           for l in range(L)] for t in range(T)]
    flat = np.concatenate([xs[t][l].ravel() for t in range(T) for l in range(L)])
    xd = act_tensor(flat, x_dtype)
    ws = lq.workspace(layers, M, T=T)
    nbd = max(1, min(T, 8, 16 // M))
    n_units = -(-T // nbd) * L
    rounds = -(-n_units // 96)
    lq.lq_probe_enable(True)
    try:
        y = lq.lq_loop_stack(xd, layers, T, lq.LQ_OPEN, M=M, ws=ws)
        torch.cuda.synchronize()
        probe = lq.lq_probe_read()
    finally:
        lq.lq_probe_enable(False)
    assert probe["rotate_quantize"][1] == rounds and probe["gemv"][1] == rounds, probe
    yh = host(y)
    off = 0
    for t in range(T):
        for l in range(L):
            lin, mp = lins[l % nl], params[l % nl]
            n = M * lin.N
            yg = yh[off:off + n].reshape(M, lin.N)
            off += n
            q8, _, s = lq.lq_quantize_act(act_tensor(xs[t][l], x_dtype), dev(mp.P1),
                                          dev(mp.P2), float(mp.las[t]), a_bits)
            torch.cuda.synchronize()
            linear_parity(yg, xs[t][l], built[l % nl][1], t, host(q8), host(s),
                          built[l % nl][0].w_flips)


def test_loop_stack_open_more_than_eight_loops():
    """T = 11 loops with a full-size workspace: launches of 8 and 3 loops, each
    loop with its own LAS clip, checked against the oracle loop by loop."""
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    (lin,) = wl.linears
    T = 11
    mp.las = np.random.default_rng(11).uniform(0.7, 1.0, T).astype(np.float32)
    layer, ol = make_layer(mp, wl.a_bits)
    M = wl.M
    xs = [synth.loop_input(wl, lin, t, rows=np.arange(M)) for t in range(T)]
    xd = act_tensor(np.concatenate([x.ravel() for x in xs]), wl.x_dtype)
    ws = lq.workspace([layer], M, T=T)
    y = host(lq.lq_loop_stack(xd, [layer], T, lq.LQ_OPEN, M=M, ws=ws))
    torch.cuda.synchronize()
    for t in range(T):
        q8, _, s = lq.lq_quantize_act(act_tensor(xs[t], wl.x_dtype), dev(mp.P1), dev(mp.P2),
                                      float(mp.las[t]), wl.a_bits)
        torch.cuda.synchronize()
        linear_parity(y[t * M * lin.N:(t + 1) * M * lin.N].reshape(M, lin.N), xs[t], ol, t,
                      host(q8), host(s), layer.w_flips)


def _slt_params(mp, T, seed):
    """Loop-dependent copies of a module for SLT: per loop its own orthogonal
    P1_t, P2_t and weight W_t (the shared weight plus a small loop-specific change)."""
    rng = np.random.default_rng(seed)
    out = []
    for t in range(T):
        q = copy.copy(mp)
        a, b = mp.P1.shape[0], mp.P2.shape[0]
        q.P1 = np.linalg.qr(rng.standard_normal((a, a)))[0].astype(np.float32)
        q.P2 = np.linalg.qr(rng.standard_normal((b, b)))[0].astype(np.float32)
        q.W = (mp.W + 0.002 * rng.standard_normal(mp.W.shape)).astype(np.float32)
        out.append(q)
    return out


@pytest.mark.parametrize("wl,M,sel", [(synth.MLP, 256, 1), (synth.TINY, 64, 0)],
                         ids=["mlp_up_selected", "tiny"])
def test_loop_stack_slt_open(wl, M, sel):
    """SLT serving in open mode: module `sel` has its own transform and weight at
    every loop, the others share theirs (and keep sharing launches across loops);
    every step is checked against the oracle's SLT schedule."""
    params = synth.module_params(wl)
    T, L = wl.T, len(wl.linears)
    built = [make_layer(mp, wl.a_bits) for mp in params]
    own = [make_layer(q, wl.a_bits) for q in _slt_params(params[sel], T, 7)]
    tl = [[own[t] if l == sel else built[l] for l in range(L)] for t in range(T)]
    xs, flat = _stack_inputs(wl, M)
    xd = act_tensor(flat, wl.x_dtype)
    y = host(lq.lq_loop_stack_slt(xd, [[h[0] for h in row] for row in tl], lq.LQ_OPEN, M=M))
    torch.cuda.synchronize()
    ys_or = O.loop_stack_slt_open(xs, [[h[1] for h in row] for row in tl], T)
    off = 0
    for t in range(T):
        for l, lin in enumerate(wl.linears):
            n = M * lin.N
            yg = y[off:off + n].reshape(M, lin.N)
            off += n
            layer, ol = tl[t][l]
            q8, _, sc = lq.lq_quantize_act(act_tensor(xs[t][l], wl.x_dtype), dev(ol.P1),
                                           dev(ol.P2), float(ol.las[t]), wl.a_bits)
            torch.cuda.synchronize()
            y_or, _ = linear_parity(yg, xs[t][l], ol, t, host(q8), host(sc), layer.w_flips)
            np.testing.assert_allclose(y_or, ys_or[t][l], rtol=1e-12, atol=0)


def test_loop_stack_slt_chain_tiny():
    """SLT serving in chain mode: the tiny shared linear selected, a different
    transform and weight at each of its 4 loops, y_t feeding loop t + 1."""
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    (lin,) = wl.linears
    own = [make_layer(q, 4) for q in _slt_params(mp, wl.T, 9)]
    x0 = synth.loop_input(wl, lin, 0)
    y = host(lq.lq_loop_stack_slt(dev(x0), [[h[0]] for h in own], lq.LQ_CHAIN, M=wl.M))
    torch.cuda.synchronize()
    ys = O.loop_stack_slt_chain(x0, [[h[1]] for h in own], wl.T)
    for t in range(wl.T):
        check_gemm(y[t * wl.M * lin.N:(t + 1) * wl.M * lin.N].reshape(wl.M, lin.N), ys[t][0],
                   what=f"slt chain t={t}")


@pytest.mark.parametrize("mode", ["open", "chain"])
def test_loop_stack_slt_decode(mode):
    """SLT serving at decode size (4 tokens, two 2048 x 2048 modules, T = 4,
    module 0 selected with its own transform and weight per loop): open mode
    runs every unit (the selected module one loop per unit, the shared one all
    four loops in one) in one grouped quantize and one grouped GEMV launch,
    chain mode runs every step in the persistent kernel with the per-step
    handles; each step against the oracle on its actual input."""
    M, T = 4, 4
    lins = (synth.Linear("s0", 2048, 2048, 32, 64, 0), synth.Linear("s1", 2048, 2048, 32, 64, 1))
    wl = synth.Workload("slt_decode", M=M, T=T, linears=lins, a_bits=8, outlier_frac=0.02,
                        outlier_mult=20.0, x_dtype="bf16", description="SLT decode stack")
    params = synth.module_params(wl)
    shared = make_layer(params[1], 8)
    own = [make_layer(q, 8) for q in _slt_params(params[0], T, 11)]
    tl = [[own[t], shared] for t in range(T)]
    handles = [[h[0] for h in row] for row in tl]
    lq.lq_probe_enable(True)
    try:
        if mode == "open":
            xs, flat = _stack_inputs(wl, M)
            y = host(lq.lq_loop_stack_slt(act_tensor(flat, "bf16"), handles, lq.LQ_OPEN, M=M))
        else:
            x0 = synth.loop_input(wl, lins[0], 0)
            y = host(lq.lq_loop_stack_slt(act_tensor(x0, "bf16"), handles, lq.LQ_CHAIN, M=M))
        torch.cuda.synchronize()
        probe = lq.lq_probe_read()
    finally:
        lq.lq_probe_enable(False)
    if mode == "open":
        assert probe["rotate_quantize"][1] == 1 and probe["gemv"][1] == 1, probe
    else:
        assert probe["chain_decode"][1] == 1 and probe["gemv"][1] == 0, probe
    off = 0
    xin, xdt = (None, "bf16") if mode == "open" else (x0, "bf16")
    for t in range(T):
        for l in range(2):
            layer, ol = tl[t][l]
            yg = y[off:off + M * 2048].reshape(M, 2048)
            off += M * 2048
            x = xs[t][l] if mode == "open" else xin
            q8, _, sc = lq.lq_quantize_act(act_tensor(x, xdt), dev(ol.P1), dev(ol.P2),
                                           float(ol.las[t]), 8)
            torch.cuda.synchronize()
            linear_parity(yg, x, ol, t, host(q8), host(sc), layer.w_flips)
            if mode == "chain":
                xin, xdt = yg, "f32"


def test_loop_stack_slt_rejects_shape_mismatch():
    wl = synth.MLP
    params = synth.module_params(wl)
    gate, _ = make_layer(params[0], 4)
    down, _ = make_layer(params[2], 4)
    x = torch.zeros(2 * 64 * 2048, device="cuda")
    with pytest.raises(lq.LQError) as e:
        lq.lq_loop_stack_slt(x, [[gate], [down]], lq.LQ_OPEN, M=64)
    assert e.value.status == lq.LQ_ERR_SHAPE


def test_loop_stack_chain_tiny():
    """Chain mode feeds y_{t} back as x_{t+1} (T = 4 loops of one shared layer)."""
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    (lin,) = wl.linears
    layer, ol = make_layer(mp, 4)
    x0 = synth.loop_input(wl, lin, 0)
    y = host(lq.lq_loop_stack(dev(x0), [layer], wl.T, lq.LQ_CHAIN, M=wl.M))
    torch.cuda.synchronize()
    ys = O.loop_stack_chain(x0, [ol], wl.T)
    for t in range(wl.T):
        check_gemm(y[t * wl.M * lin.N:(t + 1) * wl.M * lin.N].reshape(wl.M, lin.N), ys[t][0],
                   what=f"chain t={t}")


def _chain_decode_case(M, a_bits, x_dtype, T, wide=False):
    """Three chained linears 2048 -> 1024 -> 3072 -> 2048 (factors 32x64,
    32x32, 32x96), or with `wide` 4096 -> 2048 -> 1024 -> 4096 (64x64, 32x64,
    32x32), T loops with their own clips; returns the built layers, the first
    input and the GPU outputs of the chain-mode stack with the probe counts."""
    if wide:
        lins = (synth.Linear("w0", 4096, 2048, 64, 64, 0),
                synth.Linear("w1", 2048, 1024, 32, 64, 1),
                synth.Linear("w2", 1024, 4096, 32, 32, 2))
    else:
        lins = (synth.Linear("c0", 2048, 1024, 32, 64, 0),
                synth.Linear("c1", 1024, 3072, 32, 32, 1),
                synth.Linear("c2", 3072, 2048, 32, 96, 2))
    wl = synth.Workload(f"chain_M{M}", M=M, T=T, linears=lins, a_bits=a_bits,
                        outlier_frac=0.02, outlier_mult=20.0, x_dtype=x_dtype,
                        description="chain-mode decode stack")
    params = synth.module_params(wl)
    rng = np.random.default_rng(M + T)
    for mp in params:
        mp.las = rng.uniform(0.7, 1.0, T).astype(np.float32)
    built = [make_layer(mp, a_bits) for mp in params]
    x0 = synth.loop_input(wl, lins[0], 0)
    lq.lq_probe_enable(True)
    try:
        y = lq.lq_loop_stack(act_tensor(x0, x_dtype), [b[0] for b in built], T, lq.LQ_CHAIN, M=M)
        torch.cuda.synchronize()
        probe = lq.lq_probe_read()
    finally:
        lq.lq_probe_enable(False)
    return lins, params, built, x0, host(y), probe


@pytest.mark.parametrize("M,a_bits,x_dtype,T,wide", [(1, 8, "bf16", 4, False),
                                                     (3, 4, "f32", 4, False),
                                                     (4, 8, "bf16", 4, False),
                                                     (4, 4, "bf16", 43, False),
                                                     (2, 8, "bf16", 4, True)])
def test_loop_stack_chain_decode_persistent(M, a_bits, x_dtype, T, wide):
    """Decode-sized chain mode runs every step in the persistent kernel (one
    launch per 128 steps; the quantize and the GEMV of a step handed over
    through step counters): each step's output against the oracle applied to
    the step's actual input (the stack's input, then the previous step's
    float32 output).  Factor shapes 32x32 to 64x64 (K = 1024 to 4096)."""
    lins, params, built, x0, y, probe = _chain_decode_case(M, a_bits, x_dtype, T, wide)
    L = len(lins)
    n_launch = -(-(T * L) // 128)
    assert probe["chain_decode"][1] == n_launch and probe["gemv"][1] == 0, probe
    off = 0
    xin, xin_dtype = x0, x_dtype
    for t in range(T):
        for l in range(L):
            lin, mp = lins[l], params[l]
            n = M * lin.N
            yg = y[off:off + n].reshape(M, lin.N)
            off += n
            q8, _, s = lq.lq_quantize_act(act_tensor(xin, xin_dtype), dev(mp.P1), dev(mp.P2),
                                          float(mp.las[t]), a_bits)
            torch.cuda.synchronize()
            linear_parity(yg, xin, built[l][1], t, host(q8), host(s), built[l][0].w_flips)
            xin, xin_dtype = yg, "f32"


def test_loop_stack_chain_shape_check():
    wl = synth.MLP
    params = synth.module_params(wl)
    layers = [make_layer(mp, 4)[0] for mp in params[:2]]  # gate -> up: 5632 != 2048
    x = torch.zeros((64, 2048), device="cuda")
    with pytest.raises(lq.LQError) as e:
        lq.lq_loop_stack(x, layers, 2, lq.LQ_CHAIN, M=64)
    assert e.value.status == lq.LQ_ERR_SHAPE


def test_loop_stack_inside_caller_capture():
    """When the caller's stream is capturing, the stack records into that capture."""
    wl = synth.TINY
    (mp,) = synth.module_params(wl)
    layer, _ = make_layer(mp, 4)
    xs, flat = _stack_inputs(wl, wl.M)
    xd = act_tensor(flat, wl.x_dtype)
    ref = lq.lq_loop_stack(xd, [layer], wl.T, lq.LQ_OPEN, M=wl.M)
    y = torch.zeros_like(ref)
    ws = lq.workspace([layer], wl.M)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        lq.lq_loop_stack(xd, [layer], wl.T, lq.LQ_OPEN, M=wl.M, y=y, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, ref)


def test_calib_block_full_size_sampled_rows():
    """Full 262144-token calibration block: every (module, loop) at full size,
    checked on sampled rows (rows are independent)."""
    wl = synth.CALIB_BLOCK
    params = synth.module_params(wl)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(wl.M, 192, replace=False))
    rows[0], rows[-1] = 0, wl.M - 1
    rows_d = torch.from_numpy(rows).cuda()
    for l, (lin, mp) in enumerate(zip(wl.linears, params)):
        layer, ol = make_layer(mp, wl.a_bits)
        for t in ((0, 3) if l % 2 else (1, 2)):
            x = synth.device_loop_input(wl, lin, t)
            y = lq.lq_loop_linear(x, layer, t)
            ys = host(y[rows_d])
            xs = x[rows_d].float().cpu().numpy()
            del y
            q8, _, s = lq.lq_quantize_act(x[rows_d].contiguous(), dev(mp.P1), dev(mp.P2),
                                          float(mp.las[t]), wl.a_bits)
            torch.cuda.synchronize()
            linear_parity(ys, xs, ol, t, host(q8), host(s), layer.w_flips)
            del x
        lq.lq_check_device()


def test_calib_block_stack_full_size_sampled_rows():
    """The benchmark's headline step at full size: lq_loop_stack in open mode
    over the 7 shared linears x T = 4 loops on M = 262144 tokens, with the
    workspace that batches the 4 loops of a linear into one quantize and one
    GEMM launch (1048576 rows per launch).  Every (module, loop) output is
    checked against the oracle on sampled rows (rows are independent): the
    first and last rows, rows at 128-row tile and 256-row block edges, and
    random rows."""
    wl = synth.CALIB_BLOCK
    params = synth.module_params(wl)
    M, T = wl.M, wl.T
    built = [make_layer(mp, wl.a_bits) for mp in params]
    layers = [b[0] for b in built]
    rng = np.random.default_rng(17)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, M // 2 - 1, M // 2, M - 129,
                                      M - 128, M - 1], rng.choice(M, 53, replace=False)]))
    rows_d = torch.from_numpy(rows).cuda()
    sum_k = sum(lin.K for lin in wl.linears)
    sum_n = sum(lin.N for lin in wl.linears)
    x = torch.empty(T * M * sum_k, dtype=torch.bfloat16, device="cuda")
    off = 0
    for t in range(T):
        for lin in wl.linears:
            x[off:off + M * lin.K] = synth.device_loop_input(wl, lin, t).reshape(-1)
            off += M * lin.K
    y = torch.empty(T * M * sum_n, dtype=torch.float32, device="cuda")
    ws = lq.workspace(layers, M, T=T)
    lq.lq_loop_stack(x, layers, T, lq.LQ_OPEN, M=M, y=y, ws=ws)
    torch.cuda.synchronize()
    lq.lq_check_device()
    del ws
    xo = yo = 0
    for t in range(T):
        for l, (lin, mp) in enumerate(zip(wl.linears, params)):
            xs = x[xo:xo + M * lin.K].view(M, lin.K)[rows_d].contiguous()
            ys = host(y[yo:yo + M * lin.N].view(M, lin.N)[rows_d])
            xo += M * lin.K
            yo += M * lin.N
            q8, _, s = lq.lq_quantize_act(xs, dev(mp.P1), dev(mp.P2), float(mp.las[t]),
                                          wl.a_bits)
            torch.cuda.synchronize()
            linear_parity(ys, xs.float().cpu().numpy(), built[l][1], t, host(q8), host(s),
                          built[l][0].w_flips)
    del x, y
    for layer, _ in built:
        layer.free()
    torch.cuda.empty_cache()
