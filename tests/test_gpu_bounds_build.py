"""The bounds-check build (kernels compiled with -DLQ_BOUNDS_CHECK test each
checked store index against the extent it writes, skip and record a violation)
runs the path's kernels on small cases of every kind (fused rotation, its
warp-specialised and few-row forms, quantize-only, the GEMM with its weight
operand, the decode GEMV, the loop driver in open and chain mode, CTA and the
trajectory Hessian); lq_check_device must report no index out of range.  The
library is loaded in a child process (one CUDA library per process)."""
import os
import subprocess
import sys

import pytest

from bit_ptq_looped_b200 import build as B

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, ROOT)
import numpy as np, torch
from bit_ptq_looped_b200 import lq, synth
lq.lib()
assert any('liblq_bounds.so' in l for l in open('/proc/self/maps')), 'bounds build not mapped'
dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()

def layer_of(wl, a_bits=4):
    out = []
    for mp in synth.module_params(wl):
        Q1 = lq.lq_inverse_transpose(mp.P1).cuda(); Q2 = lq.lq_inverse_transpose(mp.P2).cuda()
        wq = lq.lq_pack_weights(lq.lq_fold_weights(dev(mp.W), Q1, Q2))
        out.append(lq.lq_layer_create(wq, dev(mp.P1), dev(mp.P2), mp.las, a_bits))
    return out

# open and chain stacks (tiny), open stack with loop batching (MLP, 200 rows)
tiny = layer_of(synth.TINY)
xs = [synth.loop_input(synth.TINY, synth.TINY.linears[0], t) for t in range(4)]
lq.lq_loop_stack(dev(np.concatenate([x.ravel() for x in xs])), tiny, 4, lq.LQ_OPEN, M=64)
lq.lq_loop_stack(dev(xs[0]), tiny, 4, lq.LQ_CHAIN, M=64)
mlp = layer_of(synth.MLP)
M = 200
xm = np.concatenate([synth.loop_input(synth.MLP, lin, t, rows=np.arange(M)).ravel()
                     for t in range(4) for lin in synth.MLP.linears])
lq.lq_loop_stack(dev(xm).to(torch.bfloat16), mlp, 4, lq.LQ_OPEN, M=M)
# decode stack (concurrent GEMV chains), W4A8
dec = layer_of(synth.decode_workload(4, 2048, 8), 8)
xd = np.concatenate([synth.loop_input(synth.decode_workload(4, 2048, 8),
                                      synth.decode_workload(4, 2048, 8).linears[0], t).ravel()
                     for t in range(4)])
lq.lq_loop_stack(dev(xd).to(torch.bfloat16), dec, 4, lq.LQ_OPEN, M=4)
# warp-specialised rotation (32 x 64 and 64 x 88), quantize-only, few-row rotation
rng = np.random.default_rng(0)
for (a, b), rows in (((32, 64), 2405), ((64, 88), 597)):
    P1 = np.linalg.qr(rng.standard_normal((a, a)))[0].astype(np.float32)
    P2 = np.linalg.qr(rng.standard_normal((b, b)))[0].astype(np.float32)
    x = rng.standard_normal((rows, a * b)).astype(np.float32)
    lq.lq_quantize_act(dev(x), dev(P1), dev(P2), 0.9, 4, want_codes4=True)
    lq.lq_quantize_act(dev(x[:3]), dev(P1), dev(P2), 0.9, 8)
lq.lq_quantize_act(dev(rng.standard_normal((257, 256)).astype(np.float32)), None, None, 0.8, 4)
# CTA transitions in chain mode, trajectory Hessian
d = 256
cta = lq.lq_cta_create(dev(0.05 * rng.standard_normal((d, 8)).astype(np.float32)),
                       dev(0.05 * rng.standard_normal((d, 8)).astype(np.float32)),
                       dev(np.ones((3, d), np.float32)), dev(np.zeros((3, d), np.float32)),
                       [0.5, 0.5, 0.5])
lq.lq_loop_stack_cta(dev(xs[0]), tiny, 4, cta, M=64)
xh = dev(synth.round_bf16(rng.standard_normal((3 * 100, 384)).astype(np.float32))).to(torch.bfloat16)
lq.lq_trajectory_hessian(xh, 3, M=100)
torch.cuda.synchronize()
lq.lq_check_device()
print('bounds build: no index out of range')
""".replace("ROOT", repr(ROOT))


def test_kernels_stay_in_range_under_the_bounds_check_build():
    lib = B.build_bounds_checked()
    env = dict(os.environ, LQ_LIB_PATH=lib)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, (r.stdout + r.stderr)[-3000:]
    assert "no index out of range" in r.stdout
