"""Thin ctypes binding of libparo.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: tensors are checked for dtype/device/contiguity and
their data pointers are handed to the library together with torch's current
CUDA stream. If the library is missing the import fails loudly; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libparo.so")

PARO_OK = 0
_STATUS = {0: "PARO_OK", 1: "PARO_ERR_ARG", 2: "PARO_ERR_UNSUPPORTED", 3: "PARO_ERR_CUDA", 4: "PARO_ERR_DEVICE"}

_lib: Optional[ctypes.CDLL] = None

_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "paro_rot_create": [ctypes.POINTER(_vp), _i64, _int, _int, _int, _vp, _vp, _vp],
    "paro_rot_destroy": [_vp],
    "paro_rotate": [_vp, _vp, _vp, _i64, _vp],
    "paro_pack_size": [_i64, _i64, ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(_sz)],
    "paro_pack_weights": [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp],
    "paro_dequant": [_vp, _vp, _vp, _i64, _i64, _vp, _vp],
    "paro_quantize_weights": [_vp, _vp, _i64, _vp, _vp, _vp, _vp],
    "paro_linear_workspace_size": [_i64, _i64, _i64, ctypes.POINTER(_sz)],
    "paro_linear": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp],
    "paro_linear_bias": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _sz, _vp],
    "paro_linear_noalloc": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp],
    "paro_pack_size_ex": [_i64, _i64, _int, ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(_sz)],
    "paro_pack_weights_ex": [_vp, _vp, _vp, _i64, _i64, _int, _vp, _vp, _vp, _vp],
    "paro_dequant_ex": [_vp, _vp, _vp, _i64, _i64, _int, _vp, _vp],
    "paro_linear_ex": [_vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _i64, _i64, _i64, _vp, _sz, _vp],
    "paro_linear_partial": [_vp, _vp, _vp, _vp, _vp, _int, _vp, _i64, _i64, _i64, _vp, _sz, _vp],
    "paro_finalize": [_vp, _vp, _vp, _i64, _i64, _vp],
    "paro_rotate_once": [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _int, _int, _int, _vp],
    "paro_linear_once": [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _vp],
    "paro_fault_status": [ctypes.POINTER(_int), _int],
    "paro_check_wait_timeout": [ctypes.c_uint32, _vp],
    "paro_last_error": [],
}


class ParoError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libparo.so (built in-tree by rotated_w4_linear_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m rotated_w4_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_char_p if name == "paro_last_error" else ctypes.c_int
        _lib = L
    return _lib


def _check(fn: str, st: int) -> None:
    if st != PARO_OK:
        raise ParoError(fn, st, lib().paro_last_error().decode())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device: Optional[torch.device] = None) -> int:
    """Raw cudaStream_t: the given stream, else the current stream of the
    tensor's device (read without building a torch Stream object, which
    costs a few microseconds per call on the decode path)."""
    if stream is None:
        idx = device.index if device is not None and device.index is not None else torch.cuda.current_device()
        if _raw_stream is not None:
            return int(_raw_stream(idx))
        stream = torch.cuda.current_stream(idx)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


class Rotation:
    """Owner of a paro_rot handle (device-resident prepared rotation)."""

    def __init__(self, pairs: np.ndarray, theta: np.ndarray, alpha: np.ndarray, group: int = 128):
        pairs = np.ascontiguousarray(pairs, dtype=np.int16)
        theta = np.ascontiguousarray(theta, dtype=np.float32)
        alpha = np.ascontiguousarray(alpha, dtype=np.float32)
        K = int(pairs.shape[0]) if pairs.ndim == 4 else 0
        P = int(pairs.shape[2]) if K else 0
        self.in_features = int(alpha.shape[0])
        self.K, self.P, self.group = K, P, int(group)
        h = _vp()
        _check("paro_rot_create", lib().paro_rot_create(
            ctypes.byref(h), self.in_features, group, K, P,
            pairs.ctypes.data if K else None, theta.ctypes.data if K else None, alpha.ctypes.data))
        self.handle = h

    def close(self) -> None:
        if getattr(self, "handle", None) is not None and self.handle.value:
            _check("paro_rot_destroy", lib().paro_rot_destroy(self.handle))
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def paro_rot_create(pairs, theta, alpha, group: int = 128) -> Rotation:
    return Rotation(pairs, theta, alpha, group)


def paro_rotate(rot: Rotation, X: torch.Tensor, Xr: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if Xr is None:
        Xr = torch.empty_like(X)
    _dev(X, torch.float16, "X"), _dev(Xr, torch.float16, "Xr")
    if X.shape != Xr.shape or X.dim() != 2 or X.shape[1] != rot.in_features:
        raise ValueError("X/Xr must be [tokens][in_features]")
    _check("paro_rotate", lib().paro_rotate(rot.handle, X.data_ptr(), Xr.data_ptr(), X.shape[0], _stream(stream, X.device)))
    return Xr


def paro_fault_status(clear: bool = False) -> int:
    """0, or the code of a bounded in-kernel wait that ran out (synchronous)."""
    c = _int()
    _check("paro_fault_status", lib().paro_fault_status(ctypes.byref(c), 1 if clear else 0))
    return c.value


def paro_check_wait_timeout(limit_us: int = 1000, stream=None) -> None:
    """Enqueue the self-test kernel whose bounded wait runs out (code 6)."""
    _check("paro_check_wait_timeout", lib().paro_check_wait_timeout(int(limit_us), _stream(stream)))


def paro_pack_size(in_features: int, out_features: int, group: int = 128):
    q, s, z = _sz(), _sz(), _sz()
    if group == 128:
        _check("paro_pack_size", lib().paro_pack_size(in_features, out_features, ctypes.byref(q), ctypes.byref(s),
                                                      ctypes.byref(z)))
    else:
        _check("paro_pack_size_ex", lib().paro_pack_size_ex(in_features, out_features, group, ctypes.byref(q),
                                                            ctypes.byref(s), ctypes.byref(z)))
    return q.value, s.value, z.value


def _any(t, dtype, name) -> int:
    """Data pointer of a contiguous tensor on the device or on the host."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous {dtype} tensor")
    return t.data_ptr()


def paro_pack_weights(q: torch.Tensor, s: torch.Tensor, z: torch.Tensor, stream=None, device=None,
                      group: int = 128):
    """Logical (q uint8 [out][in], s fp16 [out][in/group], z uint8
    [out][in/group]), on the device or on the host -> device format
    (qweight, scales, zeros) as uint8 tensors on `device` (default: q's
    device, else the current one)."""
    out_f, in_f = q.shape
    qb, sb, zb = paro_pack_size(in_f, out_f, group)
    dev = device or (q.device if q.is_cuda else torch.device("cuda", torch.cuda.current_device()))
    qw = torch.empty(qb, dtype=torch.uint8, device=dev)
    sp = torch.empty(sb, dtype=torch.uint8, device=dev)
    zp = torch.empty(zb, dtype=torch.uint8, device=dev)
    _check("paro_pack_weights_ex", lib().paro_pack_weights_ex(
        _any(q, torch.uint8, "q"), _any(s, torch.float16, "s"), _any(z, torch.uint8, "z"), in_f, out_f, group,
        qw.data_ptr(), sp.data_ptr(), zp.data_ptr(), _stream(stream, qw.device)))
    return qw, sp, zp


def paro_dequant(qw, sp, zp, in_features: int, out_features: int, stream=None, group: int = 128) -> torch.Tensor:
    W = torch.empty((out_features, in_features), dtype=torch.float16, device=qw.device)
    _check("paro_dequant_ex", lib().paro_dequant_ex(_dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"),
                                                    _dev(zp, torch.uint8, "zeros"), in_features, out_features, group,
                                                    W.data_ptr(), _stream(stream)))
    return W


def paro_quantize_weights(rot: Rotation, W: torch.Tensor, stream=None):
    """W fp16 [out][in] -> (q uint8 [out][in], s fp16 [out][G], z uint8 [out][G]) of T W,
    G = in / the handle's group size."""
    out_f, in_f = W.shape
    G = in_f // rot.group
    q = torch.empty((out_f, in_f), dtype=torch.uint8, device=W.device)
    s = torch.empty((out_f, G), dtype=torch.float16, device=W.device)
    z = torch.empty((out_f, G), dtype=torch.uint8, device=W.device)
    _check("paro_quantize_weights", lib().paro_quantize_weights(
        rot.handle, _dev(W, torch.float16, "W"), out_f, q.data_ptr(), s.data_ptr(), z.data_ptr(), _stream(stream)))
    return q, s, z


def paro_linear_workspace_size(tokens: int, in_features: int, out_features: int) -> int:
    b = _sz()
    _check("paro_linear_workspace_size", lib().paro_linear_workspace_size(tokens, in_features, out_features, ctypes.byref(b)))
    return b.value


def workspace(tokens: int, in_features: int, out_features: int, device=None) -> torch.Tensor:
    """A zero-filled workspace of the size paro_linear needs (allocated by torch)."""
    n = paro_linear_workspace_size(tokens, in_features, out_features)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def paro_linear(rot: Optional[Rotation], X: torch.Tensor, qw, sp, zp, out_features: int,
                Y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    T, in_f = X.shape
    if Y is None:
        Y = torch.empty((T, out_features), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(T, in_f, out_features, X.device)
    _check("paro_linear", lib().paro_linear(
        rot.handle if rot is not None else None, _dev(X, torch.float16, "X"),
        _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"), _dev(zp, torch.uint8, "zeros"),
        _dev(Y, torch.float16, "Y"), T, in_f, out_features, _dev(ws, torch.uint8, "workspace"), ws.numel(),
        _stream(stream, X.device)))
    return Y


def paro_linear_bias(rot: Optional[Rotation], X: torch.Tensor, qw, sp, zp, bias: Optional[torch.Tensor],
                     out_features: int, Y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """paro_linear + bias (fp16 [out_features] CUDA tensor, or None)."""
    T, in_f = X.shape
    if Y is None:
        Y = torch.empty((T, out_features), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(T, in_f, out_features, X.device)
    b = None
    if bias is not None:
        if bias.numel() != out_features:
            raise ValueError("bias must have out_features elements")
        b = _dev(bias, torch.float16, "bias")
    _check("paro_linear_bias", lib().paro_linear_bias(
        rot.handle if rot is not None else None, _dev(X, torch.float16, "X"),
        _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"), _dev(zp, torch.uint8, "zeros"), b,
        _dev(Y, torch.float16, "Y"), T, in_f, out_features, _dev(ws, torch.uint8, "workspace"), ws.numel(),
        _stream(stream, X.device)))
    return Y


def paro_rotate_once(X: torch.Tensor, pairs, theta, alpha, group: int = 128, stream=None) -> torch.Tensor:
    """X T^-1 from (pairs, theta, alpha) without a handle (allocating, synchronous)."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int16)
    theta = np.ascontiguousarray(theta, dtype=np.float32)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    K = int(pairs.shape[0])
    P = int(pairs.shape[2]) if K else 0
    Xr = torch.empty_like(X)
    T, in_f = X.shape
    _check("paro_rotate_once", lib().paro_rotate_once(
        _dev(X, torch.float16, "X"), _dev(Xr, torch.float16, "Xr"), T, in_f, pairs.ctypes.data if K else None,
        theta.ctypes.data if K else None, alpha.ctypes.data, K, group, P, _stream(stream, X.device)))
    return Xr


def paro_linear_once(X: torch.Tensor, pairs, theta, alpha, qw, sp, zp, out_features: int,
                     stream=None) -> torch.Tensor:
    """Y = (X T^-1) w_hat^T from (pairs, theta, alpha) without a handle
    (allocating, synchronous)."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int16)
    theta = np.ascontiguousarray(theta, dtype=np.float32)
    alpha = np.ascontiguousarray(alpha, dtype=np.float32)
    K = int(pairs.shape[0])
    P = int(pairs.shape[2]) if K else 0
    T, in_f = X.shape
    Y = torch.empty((T, out_features), dtype=torch.float16, device=X.device)
    _check("paro_linear_once", lib().paro_linear_once(
        _dev(X, torch.float16, "X"), pairs.ctypes.data if K else None, theta.ctypes.data if K else None,
        alpha.ctypes.data, _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"),
        _dev(zp, torch.uint8, "zeros"), _dev(Y, torch.float16, "Y"), T, in_f, out_features, K, P,
        _stream(stream, X.device)))
    return Y


def paro_linear_ex(rot: Optional[Rotation], X: torch.Tensor, qw, sp, zp, out_features: int, group: int = 128,
                   bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The layer with weights quantised in groups of `group` channels (128 or 64)."""
    T, in_f = X.shape
    if Y is None:
        Y = torch.empty((T, out_features), dtype=torch.float16, device=X.device)
    if ws is None:
        ws = workspace(T, in_f, out_features, X.device)
    b = None
    if bias is not None:
        if bias.numel() != out_features:
            raise ValueError("bias must have out_features elements")
        b = _dev(bias, torch.float16, "bias")
    _check("paro_linear_ex", lib().paro_linear_ex(
        rot.handle if rot is not None else None, _dev(X, torch.float16, "X"),
        _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"), _dev(zp, torch.uint8, "zeros"), b, group,
        _dev(Y, torch.float16, "Y"), T, in_f, out_features, _dev(ws, torch.uint8, "workspace"), ws.numel(),
        _stream(stream, X.device)))
    return Y


class ParoLinear:
    """A prepared layer for repeated calls (a decode loop): the rotation
    handle, the packed weights, the bias and a workspace are checked once
    here; a call checks only X and Y and hands raw pointers to the same C
    entry point as paro_linear_ex. The workspace is owned by the object and
    grows with the largest batch seen, so calls on one object must not
    overlap on the GPU (one stream, or events), as for paro_linear's
    workspace. The object keeps references to the tensors it was given."""

    def __init__(self, rot: Optional[Rotation], qw, sp, zp, in_features: int, out_features: int, group: int = 128,
                 bias: Optional[torch.Tensor] = None, device=None):
        if rot is not None and (rot.group != group or rot.in_features != in_features):
            raise ValueError("the rotation was prepared for another group size or input width")
        self.rot, self.in_features, self.out_features, self.group = rot, int(in_features), int(out_features), group
        self._tensors = (qw, sp, zp, bias)                 # kept alive for the pointers below
        self._h = rot.handle if rot is not None else None
        self._qw, self._sp, self._zp = _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"), \
            _dev(zp, torch.uint8, "zeros")
        self._b = None
        if bias is not None:
            if bias.numel() != out_features:
                raise ValueError("bias must have out_features elements")
            self._b = _dev(bias, torch.float16, "bias")
        self.device = qw.device if device is None else torch.device(device)
        self._ws = None
        self._ws_tokens = 0
        self._f = lib().paro_linear_ex

    def _workspace(self, T: int) -> None:
        if T > self._ws_tokens:
            self._ws = workspace(T, self.in_features, self.out_features, self.device)
            self._ws_tokens = T

    def __call__(self, X: torch.Tensor, Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = X.shape[0]
        if not X.is_cuda or X.dtype is not torch.float16 or not X.is_contiguous() or X.dim() != 2 \
                or X.shape[1] != self.in_features:
            raise TypeError(f"X must be a contiguous fp16 CUDA tensor [tokens][{self.in_features}]")
        if Y is None:
            Y = torch.empty((T, self.out_features), dtype=torch.float16, device=X.device)
        elif not Y.is_cuda or Y.dtype is not torch.float16 or not Y.is_contiguous() or Y.numel() != T * self.out_features:
            raise TypeError(f"Y must be a contiguous fp16 CUDA tensor [tokens][{self.out_features}]")
        if T > self._ws_tokens:
            self._workspace(T)
        if stream is None:
            sp = int(_raw_stream(X.get_device())) if _raw_stream is not None else _stream(None, X.device)
        else:
            sp = _stream(stream, X.device)
        st = self._f(self._h, X.data_ptr(), self._qw, self._sp, self._zp, self._b, self.group, Y.data_ptr(), T,
                     self.in_features, self.out_features, self._ws.data_ptr(), self._ws.numel(), sp)
        if st != PARO_OK:
            _check("paro_linear_ex", st)
        return Y


def paro_linear_partial(rot: Optional[Rotation], X: torch.Tensor, qw, sp, zp, out_features: int, group: int = 128,
                        Yf: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """A row-parallel rank's unrounded fp32 share of Y over its input slice."""
    T, in_f = X.shape
    if Yf is None:
        Yf = torch.empty((T, out_features), dtype=torch.float32, device=X.device)
    if ws is None:
        ws = workspace(T, in_f, out_features, X.device)
    _check("paro_linear_partial", lib().paro_linear_partial(
        rot.handle if rot is not None else None, _dev(X, torch.float16, "X"),
        _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"), _dev(zp, torch.uint8, "zeros"), group,
        _dev(Yf, torch.float32, "Yf"), T, in_f, out_features, _dev(ws, torch.uint8, "workspace"), ws.numel(),
        _stream(stream, X.device)))
    return Yf


def paro_finalize(Yf: torch.Tensor, bias: Optional[torch.Tensor] = None, Y: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """fp16(Yf + bias), one rounding."""
    T, out_f = Yf.shape
    if Y is None:
        Y = torch.empty((T, out_f), dtype=torch.float16, device=Yf.device)
    b = _dev(bias, torch.float16, "bias") if bias is not None else None
    _check("paro_finalize", lib().paro_finalize(_dev(Yf, torch.float32, "Yf"), b, _dev(Y, torch.float16, "Y"), T, out_f,
                                                _stream(stream, Yf.device)))
    return Y


def paro_linear_noalloc(rot: Optional[Rotation], X: torch.Tensor, qw, sp, zp, out_features: int,
                        Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode (tokens <= 16) with the library's static scratch: no workspace,
    no device allocation inside the call (Y is allocated here only if not given)."""
    T, in_f = X.shape
    if Y is None:
        Y = torch.empty((T, out_features), dtype=torch.float16, device=X.device)
    _check("paro_linear_noalloc", lib().paro_linear_noalloc(
        rot.handle if rot is not None else None, _dev(X, torch.float16, "X"),
        _dev(qw, torch.uint8, "qweight"), _dev(sp, torch.uint8, "scales"), _dev(zp, torch.uint8, "zeros"),
        _dev(Y, torch.float16, "Y"), T, in_f, out_features, _stream(stream, X.device)))
    return Y
