"""Thin ctypes binding of liblq.so (argument marshalling only).

Every function here forwards to the C entry point of the same name declared
in include/lq.h; all arithmetic runs in the library's CUDA kernels.  Device
buffers are torch tensors (PyTorch is used for device memory and streams
only).  There is no fallback: if the library cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# LQ_LIB_PATH selects another build of the same library (the host-sanitizer
# build in the sanitizer test); by default the in-tree liblq.so
LIB_PATH = os.environ.get("LQ_LIB_PATH") or os.path.join(HERE, "liblq.so")

LQ_OK, LQ_ERR_ARG, LQ_ERR_SHAPE, LQ_ERR_UNSUPPORTED, LQ_ERR_ALIGN = 0, 1, 2, 3, 4
LQ_ERR_CUDA, LQ_ERR_DEVICE_TIMEOUT, LQ_ERR_NOMEM, LQ_ERR_WORKSPACE = 5, 6, 7, 8
LQ_ERR_DEVICE_BOUNDS = 9
LQ_F32, LQ_BF16 = 0, 1
LQ_OPEN, LQ_CHAIN = 0, 1

STATUS_NAMES = {0: "LQ_OK", 1: "LQ_ERR_ARG", 2: "LQ_ERR_SHAPE", 3: "LQ_ERR_UNSUPPORTED",
                4: "LQ_ERR_ALIGN", 5: "LQ_ERR_CUDA", 6: "LQ_ERR_DEVICE_TIMEOUT",
                7: "LQ_ERR_NOMEM", 8: "LQ_ERR_WORKSPACE", 9: "LQ_ERR_DEVICE_BOUNDS"}

# symbol -> (restype, argtypes)
_vp, _i32, _i64, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_pp = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "lq_last_error": (ctypes.c_char_p, []),
    "lq_version": (_i32, []),
    "lq_act_scale_bytes": (_i64, [_i64, _i64]),
    "lq_quantize_act": (_i32, [_vp, _i32, _i64, _i64, _vp, _i32, _vp, _i32, _f32, _i32, _i32,
                               _vp, _vp, _vp, _vp]),
    "lq_fold_weights": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _i32, _vp, _vp]),
    "lq_inverse_transpose": (_i32, [_vp, _i32, _vp]),
    "lq_quantize_weights": (_i32, [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
    "lq_pack_weights": (_i32, [_vp, _i64, _i64, _i32, _i32, _pp, _vp]),
    "lq_wq_info": (_i32, [_vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64), _pp, _pp,
                          ctypes.POINTER(_i64)]),
    "lq_wq_free": (None, [_vp]),
    "lq_layer_create": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp, _i32, _i32, _pp]),
    "lq_layer_free": (None, [_vp]),
    "lq_workspace_bytes": (_i64, [_pp, _i32, _i64]),
    "lq_stack_workspace_bytes": (_i64, [_pp, _i32, _i64, _i32]),
    "lq_loop_linear": (_i32, [_vp, _i32, _i64, _vp, _i32, _vp, _vp, _i64, _vp]),
    "lq_loop_stack": (_i32, [_vp, _i32, _i64, _pp, _i32, _i32, _i32, _vp, _vp, _i64, _vp]),
    "lq_loop_stack_slt": (_i32, [_vp, _i32, _i64, _pp, _i32, _i32, _i32, _vp, _vp, _i64, _vp]),
    "lq_hessian_workspace_bytes": (_i64, [_i64, _i64, _i32]),
    "lq_trajectory_hessian": (_i32, [_vp, _i32, _i64, _i64, _i32, _vp, _i32, _vp, _i64, _vp]),
    "lq_cta_create": (_i32, [_vp, _vp, _i64, _i32, _vp, _vp, _vp, _i32, _pp]),
    "lq_cta_free": (None, [_vp]),
    "lq_cta_apply": (_i32, [_vp, _i64, _vp, _i32, _vp, _vp]),
    "lq_cta_stack_workspace_bytes": (_i64, [_pp, _i32, _i64]),
    "lq_loop_stack_cta": (_i32, [_vp, _i32, _i64, _pp, _i32, _i32, _vp, _vp, _vp, _i64, _vp]),
    "lq_check_device": (_i32, [_vp]),
    "lq_selftest_bounded_wait": (_i32, [_i64, _vp]),
    "lq_selftest_grid_wait": (_i32, [_i64, _vp, _vp]),
    "lq_loop_linear_noalloc": (_i32, [_vp, _i32, _i64, _vp, _i32, _vp, _vp]),
    "lq_probe_enable": (_i32, [_i32]),
    "lq_probe_read": (_i32, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)]),
}

PROBE_KINDS = ("rotate_quantize", "quantize", "gemm", "gemv", "weight_operand", "chain_decode")

_lib: Optional[ctypes.CDLL] = None


class LQError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load liblq.so (fails loudly if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"liblq.so is not built ({LIB_PATH}); run "
                               "`python -m bit_ptq_looped_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != LQ_OK:
        raise LQError(status, where, lib().lq_last_error().decode())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return LQ_F32
    if x.dtype == torch.bfloat16:
        return LQ_BF16
    raise ValueError(f"unsupported activation dtype {x.dtype}")


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------
def lq_quantize_act(x: torch.Tensor, P1: Optional[torch.Tensor], P2: Optional[torch.Tensor],
                    las_t: float, bits: int, group: int = 32, *,
                    codes8: Optional[torch.Tensor] = None, codes4: Optional[torch.Tensor] = None,
                    scales: Optional[torch.Tensor] = None, want_codes8: bool = True,
                    want_codes4: bool = False, stream=None):
    """Returns (codes8, codes4, scales); buffers are allocated with torch when not given."""
    M, K = x.shape
    dev = x.device
    if codes8 is None and want_codes8:
        codes8 = torch.empty((M, K), dtype=torch.int8, device=dev)
    if codes4 is None and want_codes4:
        codes4 = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((M, K // 32), dtype=torch.float32, device=dev)
    a = P1.shape[0] if P1 is not None else 0
    b = P2.shape[0] if P2 is not None else 0
    st = lib().lq_quantize_act(_dev(x, "x"), _dtype_code(x), M, K,
                               _ptr(P1), a, _ptr(P2), b, float(las_t), bits, group,
                               _ptr(codes8), _ptr(codes4), _ptr(scales), _stream(stream))
    _check(st, "lq_quantize_act")
    return codes8, codes4, scales


def lq_fold_weights(W: torch.Tensor, Q1: torch.Tensor, Q2: torch.Tensor, out=None, stream=None):
    N, K = W.shape
    if out is None:
        out = torch.empty_like(W)
    st = lib().lq_fold_weights(_dev(W, "W"), N, K, _dev(Q1, "Q1"), Q1.shape[0], _dev(Q2, "Q2"),
                               Q2.shape[0], _dev(out, "out"), _stream(stream))
    _check(st, "lq_fold_weights")
    return out


def lq_inverse_transpose(P) -> torch.Tensor:
    P = torch.as_tensor(P, dtype=torch.float32).contiguous().cpu()
    out = torch.empty_like(P)
    st = lib().lq_inverse_transpose(P.data_ptr(), P.shape[0], out.data_ptr())
    _check(st, "lq_inverse_transpose")
    return out


def lq_quantize_weights(W: torch.Tensor, bits: int = 4, group: int = 32, *, want_codes8=True,
                        want_codes4=True, stream=None):
    N, K = W.shape
    codes8 = torch.empty((N, K), dtype=torch.int8, device=W.device) if want_codes8 else None
    codes4 = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device) if want_codes4 else None
    scales = torch.empty((N, K // 32), dtype=torch.float32, device=W.device)
    st = lib().lq_quantize_weights(_dev(W, "W"), N, K, bits, group, _ptr(codes8), _ptr(codes4),
                                   _ptr(scales), _stream(stream))
    _check(st, "lq_quantize_weights")
    return codes8, codes4, scales


class PackedWeights:
    """Owner of an lq_wq handle (library-owned device memory)."""

    def __init__(self, handle: int):
        self.handle = handle

    def info(self):
        N, K, nbytes = _i64(), _i64(), _i64()
        c4, sc = ctypes.c_void_p(), ctypes.c_void_p()
        _check(lib().lq_wq_info(self.handle, ctypes.byref(N), ctypes.byref(K), ctypes.byref(c4),
                                ctypes.byref(sc), ctypes.byref(nbytes)), "lq_wq_info")
        return dict(N=N.value, K=K.value, codes4=c4.value, scales=sc.value,
                    device_bytes=nbytes.value)

    def free(self):
        if self.handle:
            lib().lq_wq_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def lq_pack_weights(W_folded: torch.Tensor, bits: int = 4, group: int = 32,
                    stream=None) -> PackedWeights:
    N, K = W_folded.shape
    h = ctypes.c_void_p()
    st = lib().lq_pack_weights(_dev(W_folded, "W"), N, K, bits, group, ctypes.byref(h),
                               _stream(stream))
    _check(st, "lq_pack_weights")
    return PackedWeights(h.value)


class _DeviceView:
    """__cuda_array_interface__ wrapper so torch can view library-owned device memory."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


def wq_tensors(wq: PackedWeights):
    """Copies of the resident packed codes (N x K/2 uint8) and steps (N x K/32 float32)."""
    info = wq.info()
    N, K = info["N"], info["K"]
    codes4 = torch.as_tensor(_DeviceView(info["codes4"], (N, K // 2), "|u1"), device="cuda")
    scales = torch.as_tensor(_DeviceView(info["scales"], (N, K // 32), "<f4"), device="cuda")
    return codes4.clone(), scales.clone()


class Layer:
    """Owner of an lq_layer handle; keeps its PackedWeights alive."""

    def __init__(self, handle: int, wq: PackedWeights, K: int, N: int, T: int):
        self.handle, self.wq, self.K, self.N, self.T = handle, wq, K, N, T

    def free(self):
        if self.handle:
            lib().lq_layer_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def lq_layer_create(wq: PackedWeights, P1: torch.Tensor, P2: torch.Tensor, las: Sequence[float],
                    a_bits: int = 4) -> Layer:
    las_h = torch.as_tensor(list(las), dtype=torch.float32).contiguous()
    h = ctypes.c_void_p()
    st = lib().lq_layer_create(wq.handle, _dev(P1, "P1"), P1.shape[0], _dev(P2, "P2"),
                               P2.shape[0], las_h.data_ptr(), las_h.numel(), a_bits,
                               ctypes.byref(h))
    _check(st, "lq_layer_create")
    info = wq.info()
    return Layer(h.value, wq, info["K"], info["N"], las_h.numel())


def _layer_array(layers: Sequence[Layer]):
    arr = (ctypes.c_void_p * len(layers))(*[l.handle for l in layers])
    return ctypes.cast(arr, _pp), arr


def lq_workspace_bytes(layers: Sequence[Layer], M: int) -> int:
    p, keep = _layer_array(layers)
    n = lib().lq_workspace_bytes(p, len(layers), M)
    if n < 0:
        raise ValueError("invalid layers")
    return n


def lq_stack_workspace_bytes(layers: Sequence[Layer], M: int, T: int) -> int:
    p, keep = _layer_array(layers)
    n = lib().lq_stack_workspace_bytes(p, len(layers), M, T)
    if n < 0:
        raise ValueError("invalid layers or T")
    return n


def workspace(layers: Sequence[Layer], M: int, device="cuda", T: Optional[int] = None) -> torch.Tensor:
    """Workspace for M tokens; with T, the size that lets open-mode lq_loop_stack
    run the T loops of a layer in one launch (lq_stack_workspace_bytes)."""
    n = lq_workspace_bytes(layers, M) if T is None else lq_stack_workspace_bytes(layers, M, T)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def lq_loop_linear(x: torch.Tensor, layer: Layer, t: int, *, y: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, layer.N), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace([layer], M, x.device)
    st = lib().lq_loop_linear(_dev(x, "x"), _dtype_code(x), M, layer.handle, t, _dev(y, "y"),
                              _dev(ws, "ws"), ws.numel(), _stream(stream))
    _check(st, "lq_loop_linear")
    return y


def lq_loop_stack(x: torch.Tensor, layers: Sequence[Layer], T: int, mode: int = LQ_OPEN, *,
                  M: int, y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                  x_dtype: Optional[int] = None, stream=None) -> torch.Tensor:
    """x: flat buffer of the T*L inputs (open) or the first input (chain); y: flat T*L outputs."""
    if y is None:
        y = torch.empty(T * M * sum(l.N for l in layers), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(layers, M, x.device, T=T if mode == LQ_OPEN else None)
    p, keep = _layer_array(layers)
    dt = _dtype_code(x) if x_dtype is None else x_dtype
    st = lib().lq_loop_stack(_dev(x, "x"), dt, M, p, len(layers), T, mode, _dev(y, "y"),
                             _dev(ws, "ws"), ws.numel(), _stream(stream))
    _check(st, "lq_loop_stack")
    return y


def lq_loop_stack_slt(x: torch.Tensor, layers_tl: Sequence[Sequence[Layer]], mode: int = LQ_OPEN,
                      *, M: int, y: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, x_dtype: Optional[int] = None,
                      stream=None) -> torch.Tensor:
    """layers_tl[t][l]: the handle of module l at loop t (a shared module repeats
    its handle).  x and y as in lq_loop_stack."""
    T, L = len(layers_tl), len(layers_tl[0])
    flat = [layers_tl[t][l] for t in range(T) for l in range(L)]
    if any(len(row) != L for row in layers_tl):
        raise ValueError("every loop needs L handles")
    if y is None:
        y = torch.empty(T * M * sum(l.N for l in layers_tl[0]), dtype=torch.float32,
                        device=x.device)
    if ws is None:
        uniq = list({id(h): h for h in flat}.values())
        ws = workspace(uniq, M, x.device, T=T if mode == LQ_OPEN else None)
    p, keep = _layer_array(flat)
    dt = _dtype_code(x) if x_dtype is None else x_dtype
    st = lib().lq_loop_stack_slt(_dev(x, "x"), dt, M, p, L, T, mode, _dev(y, "y"),
                                 _dev(ws, "ws"), ws.numel(), _stream(stream))
    _check(st, "lq_loop_stack_slt")
    return y


def lq_trajectory_hessian(x: torch.Tensor, T: int, *, M: int, H: Optional[torch.Tensor] = None,
                          accumulate: bool = False, ws: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """x: the T loop inputs back to back (T*M x K bf16); returns H (K x K float32),
    H = sum_t X_t^T X_t, or H + that sum with accumulate=True."""
    K = x.numel() // max(T * M, 1) if x.dim() == 1 else x.shape[-1]
    if H is None:
        H = torch.zeros((K, K), dtype=torch.float32, device=x.device)
    if ws is None:
        n = lib().lq_hessian_workspace_bytes(M, K, T)
        if n < 0:
            raise ValueError("invalid shape")
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=x.device)
    st = lib().lq_trajectory_hessian(_dev(x, "x"), _dtype_code(x), M, K, T, _dev(H, "H"),
                                     1 if accumulate else 0, _dev(ws, "ws"), ws.numel(),
                                     _stream(stream))
    _check(st, "lq_trajectory_hessian")
    return H


class Cta:
    """Owner of an lq_cta handle (loop-transition adapter)."""

    def __init__(self, handle: int, d: int, n_trans: int):
        self.handle, self.d, self.n_trans = handle, d, n_trans

    def free(self):
        if self.handle:
            lib().lq_cta_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def lq_cta_create(U: torch.Tensor, V: torch.Tensor, a: torch.Tensor, b: torch.Tensor,
                  eta) -> Cta:
    """U, V: d x r (r <= 8); a, b: n_trans x d (device float32); eta: n_trans gates."""
    d, r = U.shape
    n = a.shape[0]
    eta_h = np.ascontiguousarray(np.asarray(eta, np.float32).reshape(n))
    h = ctypes.c_void_p()
    st = lib().lq_cta_create(_dev(U.contiguous(), "U"), _dev(V.contiguous(), "V"), d, r,
                             _dev(a.contiguous(), "a"), _dev(b.contiguous(), "b"),
                             eta_h.ctypes.data, n, ctypes.byref(h))
    _check(st, "lq_cta_create")
    return Cta(h.value, d, n)


def lq_cta_apply(h: torch.Tensor, cta: Cta, t: int, *, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    M = h.shape[0]
    if out is None:
        out = torch.empty_like(h)
    st = lib().lq_cta_apply(_dev(h, "h"), M, cta.handle, t, _dev(out, "out"), _stream(stream))
    _check(st, "lq_cta_apply")
    return out


def lq_cta_stack_workspace_bytes(layers: Sequence[Layer], M: int) -> int:
    p, keep = _layer_array(layers)
    n = lib().lq_cta_stack_workspace_bytes(p, len(layers), M)
    if n < 0:
        raise ValueError("invalid layers")
    return n


def lq_loop_stack_cta(x: torch.Tensor, layers: Sequence[Layer], T: int, cta: Cta, *, M: int,
                      y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      x_dtype: Optional[int] = None, stream=None) -> torch.Tensor:
    """Chain mode with the adapter at every loop transition; y: the T*L unadapted outputs.
    Pass the same y and ws on every call to replay the recorded schedule."""
    if y is None:
        y = torch.empty(T * M * sum(l.N for l in layers), dtype=torch.float32, device=x.device)
    p, keep = _layer_array(layers)
    if ws is None:
        ws = torch.empty(max(lq_cta_stack_workspace_bytes(layers, M), 256), dtype=torch.uint8,
                         device=x.device)
    dt = _dtype_code(x) if x_dtype is None else x_dtype
    st = lib().lq_loop_stack_cta(_dev(x, "x"), dt, M, p, len(layers), T, cta.handle,
                                 _dev(y, "y"), _dev(ws, "ws"), ws.numel(), _stream(stream))
    _check(st, "lq_loop_stack_cta")
    return y


LQ_NOALLOC_SCRATCH_BYTES = 16 << 20


def lq_loop_linear_noalloc(x: torch.Tensor, layer: Layer, t: int, *,
                           y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lq_loop_linear without a workspace (the library's fixed scratch is used;
    see include/lq.h).  ``y`` must be given by callers that cannot allocate."""
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, layer.N), dtype=torch.float32, device=x.device)
    st = lib().lq_loop_linear_noalloc(_dev(x, "x"), _dtype_code(x), M, layer.handle, t,
                                      _dev(y, "y"), _stream(stream))
    _check(st, "lq_loop_linear_noalloc")
    return y


def lq_check_device(stream=None) -> None:
    _check(lib().lq_check_device(_stream(stream)), "lq_check_device")


def lq_probe_enable(on: bool) -> None:
    _check(lib().lq_probe_enable(1 if on else 0), "lq_probe_enable")


def lq_probe_read() -> dict:
    """{kind: (total_ms, launches)} for the kernels launched since the last read."""
    ms = (ctypes.c_double * len(PROBE_KINDS))()
    cnt = (_i64 * len(PROBE_KINDS))()
    _check(lib().lq_probe_read(ms, cnt), "lq_probe_read")
    return {k: (ms[i], cnt[i]) for i, k in enumerate(PROBE_KINDS)}


def lq_selftest_bounded_wait(limit_us: int = 1000, stream=None) -> None:
    _check(lib().lq_selftest_bounded_wait(limit_us, _stream(stream)), "lq_selftest_bounded_wait")


def lq_selftest_grid_wait(scratch: torch.Tensor, limit_us: int = 1000, stream=None) -> None:
    """scratch: at least 8 bytes of device memory for the barrier's two words."""
    if scratch.numel() * scratch.element_size() < 8:
        raise ValueError("scratch needs 8 bytes")
    _check(lib().lq_selftest_grid_wait(limit_us, _dev(scratch, "scratch"), _stream(stream)),
           "lq_selftest_grid_wait")
