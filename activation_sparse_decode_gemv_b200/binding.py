"""Thin ctypes binding of libpi_ffn.so (argument marshalling only).

Every step of the decode path runs in the CUDA library; this module only
passes device pointers, sizes and the current torch stream across the C ABI.
The functions keep the C names (pi_predict, pi_sparse_ffn, ...) and take
torch CUDA tensors.  If the library is missing or fails to load, every entry
point raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import List, Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# PI_FFN_LIB: another build of this library (the sanitizer test's host-
# instrumented one); there is no non-CUDA implementation to fall back to
LIB_PATH = os.environ.get("PI_FFN_LIB") or os.path.join(HERE, "libpi_ffn.so")

PI_OK, PI_ERR_INVALID_ARG, PI_ERR_UNSUPPORTED, PI_ERR_MISALIGNED = 0, 1, 2, 3
PI_ERR_CUDA, PI_ERR_TIMEOUT, PI_ERR_DEVICE_STATUS, PI_ERR_WORKSPACE = 4, 5, 6, 7
PI_ACT_RELU, PI_ACT_SWIGLU = 0, 1
PI_W_F32, PI_W_F16, PI_W_INT4G32 = 0, 1, 2
PI_FFN_ACCUMULATE, PI_FFN_HOT_DENSE, PI_FFN_HOT_INDEX = 1, 2, 4
PI_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024  # device scratch of pi_decode_ffn_static

WTYPE = {"f32": PI_W_F32, "f16": PI_W_F16, "int4g32": PI_W_INT4G32}
ACT = {"relu": PI_ACT_RELU, "swiglu": PI_ACT_SWIGLU}

# every symbol the header declares
EXPORTS = ("pi_ffn_create", "pi_ffn_destroy", "pi_workspace_size", "pi_workspace_init", "pi_predict",
           "pi_sparse_ffn", "pi_decode_ffn", "pi_decode_ffn_stack", "pi_decode_ffn_static", "pi_debug_wait_fault",
           "pi_get_device_status", "pi_status_string")


class PiError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class pi_ffn_desc(C.Structure):
    _fields_ = [("d_model", C.c_int), ("d_ffn", C.c_int), ("rank", C.c_int), ("act", C.c_int),
                ("wtype", C.c_int), ("ptype", C.c_int), ("hot_prefix", C.c_int), ("hot_p_mean", C.c_float),
                ("w_up", C.c_void_p), ("w_gate", C.c_void_p), ("w_down_t", C.c_void_p),
                ("s_up", C.c_void_p), ("s_gate", C.c_void_p), ("s_down_t", C.c_void_p),
                ("b_up", C.c_void_p), ("p1", C.c_void_p), ("p2", C.c_void_p), ("p_bias", C.c_void_p)]


_lib = None


def lib() -> C.CDLL:
    """Load libpi_ffn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run activation_sparse_decode_gemv_b200/build.py "
                               "(there is no non-CUDA implementation)")
        L = C.CDLL(LIB_PATH)
        vp, i, sz = C.c_void_p, C.c_int, C.c_size_t
        L.pi_ffn_create.argtypes = [C.POINTER(pi_ffn_desc), C.POINTER(vp)]
        L.pi_ffn_destroy.argtypes = [vp]
        L.pi_ffn_destroy.restype = None
        L.pi_workspace_size.argtypes = [C.POINTER(vp), i, i, C.POINTER(sz)]
        L.pi_workspace_init.argtypes = [vp, sz, vp]
        L.pi_predict.argtypes = [vp, vp, i, vp, vp, vp, sz, vp]
        L.pi_sparse_ffn.argtypes = [vp, vp, i, vp, vp, vp, C.c_uint, vp, sz, vp]
        L.pi_decode_ffn.argtypes = [vp, vp, i, vp, vp, vp, C.c_uint, vp, sz, vp]
        L.pi_decode_ffn_stack.argtypes = [C.POINTER(vp), i, vp, i, vp, vp, C.c_uint, vp, sz, vp]
        L.pi_decode_ffn_static.argtypes = [vp, vp, vp, vp, vp, C.c_uint, vp, vp]
        L.pi_debug_wait_fault.argtypes = [i, C.c_uint]
        L.pi_get_device_status.argtypes = [vp, vp, C.POINTER(i)]
        L.pi_status_string.argtypes = [i]
        L.pi_status_string.restype = C.c_char_p
        for n in ("pi_ffn_create", "pi_workspace_size", "pi_workspace_init", "pi_predict", "pi_sparse_ffn",
                  "pi_decode_ffn", "pi_decode_ffn_stack", "pi_decode_ffn_static", "pi_debug_wait_fault",
                  "pi_get_device_status"):
            getattr(L, n).restype = C.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pi_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != PI_OK:
        raise PiError(rc, what)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


# The C ABI sees only pointers, so the binding checks what it cannot: each
# tensor's dtype, size (at least the extent the header states) and
# contiguity, then that all of them are CUDA tensors.  Null pointers and
# everything the header validates are left to the library.
def _need(t: Optional[torch.Tensor], what: str, dtype: torch.dtype, min_numel: int):
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{what}: dtype {t.dtype}, expected {dtype}")
    if t.numel() < min_numel:
        raise ValueError(f"{what}: {t.numel()} elements, the call needs at least {min_numel}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: must be contiguous")


def _on_device(**tensors: Optional[torch.Tensor]):
    for what, t in tensors.items():
        if t is not None and not t.is_cuda:
            raise ValueError(f"{what}: must be a CUDA tensor")


def _tokens(u: torch.Tensor, d: int, what: str) -> int:
    """Batch size of a [B, d] token tensor."""
    if u.dim() != 2 or u.shape[1] != d:
        raise ValueError(f"{what}: shape {tuple(u.shape)}, expected [B, {d}]")
    return u.shape[0]


def _need_ws(ws: torch.Tensor):
    if not ws.is_contiguous():
        raise ValueError("workspace: must be contiguous")


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


class FfnLayer:
    """A created pi_ffn handle plus references to the tensors it borrows."""

    def __init__(self, w_up, w_down_t, p1, p2, p_bias, *, act: str, wtype: str, d: int, f: int, r: int,
                 b_up=None, w_gate=None, s_up=None, s_gate=None, s_down_t=None, hot_prefix: int = 0,
                 hot_p_mean: float = 0.0):
        self._keep = [w_up, w_down_t, p1, p2, p_bias, b_up, w_gate, s_up, s_gate, s_down_t]
        ptype = PI_W_F32 if p1.dtype == torch.float32 else PI_W_F16
        self.desc = pi_ffn_desc(d, f, r, ACT[act], WTYPE[wtype], ptype, int(hot_prefix), float(hot_p_mean),
                                _p(w_up), _p(w_gate), _p(w_down_t), _p(s_up), _p(s_gate), _p(s_down_t),
                                _p(b_up), _p(p1), _p(p2), _p(p_bias))
        self.d, self.f, self.r, self.act, self.wtype = d, f, r, act, wtype
        self.u_dtype = torch.float32 if wtype == "f32" else torch.float16  # FFN input u
        h = C.c_void_p()
        _check(lib().pi_ffn_create(C.byref(self.desc), C.byref(h)), "pi_ffn_create")
        self.handle = h

    @classmethod
    def from_tensors(cls, lt) -> "FfnLayer":
        """From an ``inputs.LayerTensors`` already on the device."""
        return cls(lt.w_up, lt.w_down_t, lt.p1, lt.p2, lt.p_bias, act=lt.cfg.act, wtype=lt.cfg.wtype, d=lt.d, f=lt.f,
                   r=lt.r, b_up=lt.b_up, w_gate=lt.w_gate, s_up=lt.s_up, s_gate=lt.s_gate, s_down_t=lt.s_down_t,
                   hot_prefix=lt.hot_prefix, hot_p_mean=lt.hot_p_mean)

    def close(self):
        if getattr(self, "handle", None):
            lib().pi_ffn_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def pi_workspace_size(layers: Sequence[FfnLayer], max_batch: int) -> int:
    arr = (C.c_void_p * len(layers))(*[l.handle for l in layers])
    n = C.c_size_t()
    _check(lib().pi_workspace_size(arr, len(layers), int(max_batch), C.byref(n)), "pi_workspace_size")
    return n.value


def pi_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib().pi_workspace_init(_p(ws), ws.numel() * ws.element_size(), _stream(stream)), "pi_workspace_init")


def make_workspace(layers: Sequence[FfnLayer], max_batch: int, device=None) -> torch.Tensor:
    """Allocate (with torch) and zero a workspace for these layers."""
    n = pi_workspace_size(layers, max_batch)
    ws = torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))
    pi_workspace_init(ws)
    return ws


def _wsargs(ws: torch.Tensor):
    return _p(ws), ws.numel() * ws.element_size()


def pi_predict(layer: FfnLayer, u: torch.Tensor, idx: torch.Tensor, count: torch.Tensor, ws: torch.Tensor,
               stream=None):
    """u [B, d]; idx int32 [B, f] (ascending ids, row b at b*f); count int32 [B]."""
    B = _tokens(u, layer.d, "u")
    _need(u, "u", layer.u_dtype, B * layer.d)
    _need(idx, "idx", torch.int32, B * layer.f)
    _need(count, "count", torch.int32, B)
    _need_ws(ws)
    _on_device(u=u, idx=idx, count=count, workspace=ws)
    _check(lib().pi_predict(layer.handle, _p(u), B, _p(idx), _p(count), *_wsargs(ws), _stream(stream)), "pi_predict")


def pi_sparse_ffn(layer: FfnLayer, u: torch.Tensor, idx: torch.Tensor, count: torch.Tensor, y: torch.Tensor,
                  ws: torch.Tensor, flags: int = 0, stream=None):
    """u [B, d]; idx int32 [B, f] and count int32 [B] (the sets); y fp32 [B, d]."""
    B = _tokens(u, layer.d, "u")
    _need(u, "u", layer.u_dtype, B * layer.d)
    _need(idx, "idx", torch.int32, B * layer.f)
    _need(count, "count", torch.int32, B)
    _need(y, "y", torch.float32, B * layer.d)
    _need_ws(ws)
    _on_device(u=u, idx=idx, count=count, y=y, workspace=ws)
    _check(lib().pi_sparse_ffn(layer.handle, _p(u), B, _p(idx), _p(count), _p(y), int(flags), *_wsargs(ws),
                               _stream(stream)), "pi_sparse_ffn")


def pi_decode_ffn(layer: FfnLayer, u: torch.Tensor, y: torch.Tensor, ws: torch.Tensor,
                  idx: Optional[torch.Tensor] = None, count: Optional[torch.Tensor] = None, flags: int = 0,
                  stream=None):
    """u [B, d]; y fp32 [B, d]; optional idx int32 [B, f] and count int32 [B]."""
    B = _tokens(u, layer.d, "u")
    _need(u, "u", layer.u_dtype, B * layer.d)
    _need(y, "y", torch.float32, B * layer.d)
    _need(idx, "idx", torch.int32, B * layer.f)
    _need(count, "count", torch.int32, B)
    _need_ws(ws)
    _on_device(u=u, y=y, idx=idx, count=count, workspace=ws)
    _check(lib().pi_decode_ffn(layer.handle, _p(u), B, _p(y), _p(idx), _p(count), int(flags), *_wsargs(ws),
                               _stream(stream)), "pi_decode_ffn")


def pi_decode_ffn_static(layer: FfnLayer, u: torch.Tensor, y: torch.Tensor, idx: Optional[torch.Tensor] = None,
                         count: Optional[torch.Tensor] = None, flags: int = 0,
                         dev_status: Optional[torch.Tensor] = None, stream=None):
    """Batch-1 decode step on the library's static device scratch (no workspace)."""
    if u.numel() != layer.d or y.numel() != layer.d:
        raise ValueError("pi_decode_ffn_static is batch 1: u and y hold d elements")
    _need(u, "u", layer.u_dtype, layer.d)
    _need(y, "y", torch.float32, layer.d)
    _need(idx, "idx", torch.int32, layer.f)
    _need(count, "count", torch.int32, 1)
    _need(dev_status, "dev_status", torch.int32, 1)
    _on_device(u=u, y=y, idx=idx, count=count, dev_status=dev_status)
    _check(lib().pi_decode_ffn_static(layer.handle, _p(u), _p(y), _p(idx), _p(count), int(flags), _p(dev_status),
                                      _stream(stream)), "pi_decode_ffn_static")


def pi_decode_ffn_stack(layers: Sequence[FfnLayer], x: torch.Tensor, ws: torch.Tensor,
                        idx_trace: Optional[torch.Tensor] = None, count_trace: Optional[torch.Tensor] = None,
                        flags: int = 0, stream=None):
    """x fp32 [B, d] (the residual, updated in place); optional idx_trace int32
    [L, B, f_max] and count_trace int32 [L, B]."""
    if not layers:
        raise ValueError("pi_decode_ffn_stack needs at least one layer")
    B = _tokens(x, layers[0].d, "x")
    L, fmax = len(layers), max(l.f for l in layers)
    _need(x, "x", torch.float32, B * layers[0].d)
    _need(idx_trace, "idx_trace", torch.int32, L * B * fmax)
    _need(count_trace, "count_trace", torch.int32, L * B)
    _need_ws(ws)
    _on_device(x=x, idx_trace=idx_trace, count_trace=count_trace, workspace=ws)
    arr = (C.c_void_p * len(layers))(*[l.handle for l in layers])
    _check(lib().pi_decode_ffn_stack(arr, len(layers), _p(x), B, _p(idx_trace), _p(count_trace), int(flags),
                                     *_wsargs(ws), _stream(stream)), "pi_decode_ffn_stack")


def pi_debug_wait_fault(withhold_row: int = -1, limit_us: int = 0):
    """Test support: batch-1 fused launches never publish entry ``withhold_row``
    of h and wait at most ``limit_us`` (see the header); (-1, 0) restores
    normal runs."""
    _check(lib().pi_debug_wait_fault(int(withhold_row), int(limit_us)), "pi_debug_wait_fault")


def pi_get_device_status(ws: torch.Tensor, stream=None) -> int:
    code = C.c_int()
    _check(lib().pi_get_device_status(_p(ws), _stream(stream), C.byref(code)), "pi_get_device_status")
    return code.value
