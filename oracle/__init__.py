"""ctypes binding of the plain-C CPU oracle (numpy in, numpy out).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg.  The product path never imports this package.

Weight arguments follow the storage the CUDA path reads (the caller passes the
same host bytes to both): fp32 or fp16 row-major [rows x d]; int4g32 as uint8
[rows x d/2] of packed nibbles plus fp16 scales [rows x d/32].  fp16 arrays are
passed as numpy float16 (or their uint16 bit patterns).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

F32, F16, INT4G32 = 0, 1, 2
RELU, SWIGLU = 0, 1
WTYPES = {"f32": F32, "f16": F16, "int4g32": INT4G32}
ACTS = {"relu": RELU, "swiglu": SWIGLU}

_lib = None


def lib():
    global _lib
    if _lib is None:
        # PI_ORACLE_LIB: another build of this file (the sanitizer test's)
        path = os.environ.get("PI_ORACLE_LIB") or _build.build()
        L = C.CDLL(path)
        vp, ip, dp = C.c_void_p, C.c_int, C.c_void_p
        L.or_half_to_double.restype = C.c_double
        L.or_half_to_double.argtypes = [C.c_uint16]
        L.or_float_to_half.restype = C.c_uint16
        L.or_float_to_half.argtypes = [C.c_float]
        L.or_dequant_row.argtypes = [ip, ip, vp, vp, C.c_long, dp]
        L.or_predict.argtypes = [ip, ip, ip, ip, vp, vp, vp, ip, vp, ip, dp, dp, dp, vp, vp]
        L.or_neuron_phi.argtypes = [vp, vp, ip, dp]
        L.or_relu_preact.argtypes = [vp, vp, ip, dp]
        L.or_ffn_masked.argtypes = [vp, vp, ip, vp, vp, C.c_long, dp]
        L.or_ffn_dense.argtypes = [vp, vp, ip, dp]
        L.or_rmsnorm_f16.argtypes = [ip, ip, vp, vp, dp]
        L.or_stack.argtypes = [vp, ip, vp, ip, vp, vp, dp, dp, dp]
        for fn in ("or_dequant_row", "or_predict", "or_neuron_phi", "or_relu_preact", "or_ffn_masked",
                   "or_ffn_dense", "or_rmsnorm_f16", "or_stack"):
            getattr(L, fn).restype = C.c_int
        _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


def _chk(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: invalid arguments (rc={rc})")


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype=None):
    if a is None:
        return None
    a = np.asarray(a)
    if dtype is not None and a.dtype != dtype:
        if a.dtype == np.float16 and dtype == np.uint16:
            a = a.view(np.uint16)
        else:
            a = a.astype(dtype)
    return np.ascontiguousarray(a)


def _wt(a, wtype: int):
    if wtype == F32:
        return _c(a, np.float32)
    if wtype == F16:
        return _c(np.asarray(a).view(np.uint16) if np.asarray(a).dtype == np.float16 else a, np.uint16)
    return _c(a, np.uint8)


class _Ffn(C.Structure):
    _fields_ = [("d", C.c_int), ("f", C.c_int), ("act", C.c_int), ("wtype", C.c_int), ("utype", C.c_int),
                ("w_up", C.c_void_p), ("w_gate", C.c_void_p), ("w_down_t", C.c_void_p),
                ("s_up", C.c_void_p), ("s_gate", C.c_void_p), ("s_down_t", C.c_void_p),
                ("b_up", C.c_void_p)]


class _Layer(C.Structure):
    _fields_ = [("ffn", _Ffn), ("rank", C.c_int), ("ptype", C.c_int),
                ("p1", C.c_void_p), ("p2", C.c_void_p), ("p_bias", C.c_void_p)]


@dataclass
class Layer:
    """Host copy of one FFN layer and its predictor, as numpy arrays."""
    d: int
    f: int
    r: int
    act: str            # "relu" | "swiglu"
    wtype: str          # "f32" | "f16" | "int4g32"
    w_up: np.ndarray    # ReLU: W1; SwiGLU: W_up
    w_down_t: np.ndarray
    p1: np.ndarray
    p2: np.ndarray
    p_bias: np.ndarray
    b_up: Optional[np.ndarray] = None
    w_gate: Optional[np.ndarray] = None
    s_up: Optional[np.ndarray] = None
    s_gate: Optional[np.ndarray] = None
    s_down_t: Optional[np.ndarray] = None

    def __post_init__(self):
        wt = WTYPES[self.wtype]
        self._keep = dict(
            w_up=_wt(self.w_up, wt), w_down_t=_wt(self.w_down_t, wt),
            w_gate=None if self.w_gate is None else _wt(self.w_gate, wt),
            s_up=_c(self.s_up, np.uint16), s_gate=_c(self.s_gate, np.uint16), s_down_t=_c(self.s_down_t, np.uint16),
            b_up=_c(self.b_up, np.float32),
            p1=_wt(self.p1, F32 if self.ptype == F32 else F16), p2=_wt(self.p2, F32 if self.ptype == F32 else F16),
            p_bias=_c(self.p_bias, np.float32))

    @property
    def ptype(self) -> int:
        return F32 if np.asarray(self.p1).dtype == np.float32 else F16

    @property
    def utype(self) -> int:
        return F32 if self.wtype == "f32" else F16

    def _ffn(self) -> _Ffn:
        k = self._keep
        return _Ffn(self.d, self.f, ACTS[self.act], WTYPES[self.wtype], self.utype,
                    _ptr(k["w_up"]), _ptr(k["w_gate"]), _ptr(k["w_down_t"]),
                    _ptr(k["s_up"]), _ptr(k["s_gate"]), _ptr(k["s_down_t"]), _ptr(k["b_up"]))

    def _layer(self) -> _Layer:
        k = self._keep
        return _Layer(self._ffn(), self.r, self.ptype, _ptr(k["p1"]), _ptr(k["p2"]), _ptr(k["p_bias"]))


def _u(layer: Layer, u) -> np.ndarray:
    u = np.asarray(u)
    if u.ndim == 1:
        u = u[None, :]
    return _c(u, np.float32) if layer.utype == F32 else _wt(u, F16)


def half_to_double(bits: int) -> float:
    return lib().or_half_to_double(int(bits))


def float_to_half(x: float) -> int:
    return int(lib().or_float_to_half(float(np.float32(x))))


def dequant_row(layer_w: np.ndarray, scales: Optional[np.ndarray], wtype: str, d: int, row: int) -> np.ndarray:
    wt = WTYPES[wtype]
    w = _wt(layer_w, wt)
    s = _c(scales, np.uint16)
    out = np.empty(d, np.float64)
    _chk(lib().or_dequant_row(wt, d, _ptr(w), _ptr(s), row, _ptr(out)), "or_dequant_row")
    return out


def predict(layer: Layer, u):
    """-> dict(h [B,r], s [B,f], band [B,f], idx list of arrays, count [B])."""
    uu = _u(layer, u)
    B = uu.shape[0]
    d, f, r = layer.d, layer.f, layer.r
    h = np.empty((B, r)); s = np.empty((B, f)); band = np.empty((B, f))
    idx = np.empty((B, f), np.int32); cnt = np.empty(B, np.int32)
    k = layer._keep
    _chk(lib().or_predict(d, f, r, layer.ptype, _ptr(k["p1"]), _ptr(k["p2"]), _ptr(k["p_bias"]),
                          layer.utype, _ptr(uu), B, _ptr(h), _ptr(s), _ptr(band), _ptr(idx), _ptr(cnt)),
         "or_predict")
    return dict(h=h, s=s, band=band, idx=[idx[b, :cnt[b]].copy() for b in range(B)], count=cnt)


def neuron_phi(layer: Layer, u) -> np.ndarray:
    uu = _u(layer, u)
    B = uu.shape[0]
    phi = np.empty((B, layer.f))
    ffn = layer._ffn()
    _chk(lib().or_neuron_phi(C.byref(ffn), _ptr(uu), B, _ptr(phi)), "or_neuron_phi")
    return phi


def relu_preact(layer: Layer, u) -> np.ndarray:
    uu = _u(layer, u)
    B = uu.shape[0]
    pre = np.empty((B, layer.f))
    ffn = layer._ffn()
    _chk(lib().or_relu_preact(C.byref(ffn), _ptr(uu), B, _ptr(pre)), "or_relu_preact")
    return pre


def ffn_masked(layer: Layer, u, idx: Sequence[np.ndarray]) -> np.ndarray:
    """y [B,d] (double) = sum over each token's ascending id list of phi_i W2T_i."""
    uu = _u(layer, u)
    B = uu.shape[0]
    assert len(idx) == B
    width = max(1, max((len(a) for a in idx), default=1))
    buf = np.zeros((B, width), np.int32)
    cnt = np.zeros(B, np.int32)
    for b, a in enumerate(idx):
        buf[b, :len(a)] = a
        cnt[b] = len(a)
    y = np.empty((B, layer.d))
    ffn = layer._ffn()
    _chk(lib().or_ffn_masked(C.byref(ffn), _ptr(uu), B, _ptr(buf), _ptr(cnt), width, _ptr(y)), "or_ffn_masked")
    return y


def ffn_dense(layer: Layer, u) -> np.ndarray:
    uu = _u(layer, u)
    B = uu.shape[0]
    y = np.empty((B, layer.d))
    ffn = layer._ffn()
    _chk(lib().or_ffn_dense(C.byref(ffn), _ptr(uu), B, _ptr(y)), "or_ffn_dense")
    return y


def rmsnorm_f16(x) -> tuple[np.ndarray, np.ndarray]:
    """-> (u as float16 [B,d], decision margin [B])."""
    x = _c(np.atleast_2d(x), np.float32)
    B, d = x.shape
    u = np.empty((B, d), np.uint16)
    m = np.empty(B)
    _chk(lib().or_rmsnorm_f16(d, B, _ptr(x), _ptr(u), _ptr(m)), "or_rmsnorm_f16")
    return u.view(np.float16), m


def stack(layers: Sequence[Layer], x) -> dict:
    """Run the stacked decode (rmsnorm -> predict -> masked FFN -> residual)."""
    x = _c(np.atleast_2d(x), np.float32).copy()
    B, d = x.shape
    L = len(layers)
    f = layers[0].f
    arr = (_Layer * L)(*[ly._layer() for ly in layers])
    idx = np.empty((L, B, f), np.int32); cnt = np.empty((L, B), np.int32)
    y = np.empty((L, B, d)); sm = np.empty((L, B)); um = np.empty((L, B))
    _chk(lib().or_stack(arr, L, _ptr(x), B, _ptr(idx), _ptr(cnt), _ptr(y), _ptr(sm), _ptr(um)), "or_stack")
    return dict(x=x, idx=[[idx[l, b, :cnt[l, b]].copy() for b in range(B)] for l in range(L)], count=cnt,
                y=y, s_margin=sm, u_margin=um)
