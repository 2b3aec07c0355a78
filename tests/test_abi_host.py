"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every function include/pi_ffn.h declares, and rejects bad descriptions and
arguments before launching anything."""
import ctypes as C
import os
import re

import pytest

from activation_sparse_decode_gemv_b200 import binding as pb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pi_ffn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pi_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.environ.get("PI_FFN_LIB"):  # another build given: use it as is
        from activation_sparse_decode_gemv_b200 import build
        build.build()
    return pb.lib()


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(pb.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(8):
        assert pb.status_string(s) not in ("", "unknown status")
    assert pb.status_string(99) == "unknown status"


def _desc(**kw):
    base = dict(d_model=64, d_ffn=128, rank=16, act=pb.PI_ACT_RELU, wtype=pb.PI_W_F16, ptype=pb.PI_W_F16,
                hot_prefix=32, hot_p_mean=0.5, w_up=0x1000, w_gate=None, w_down_t=0x2000, s_up=None, s_gate=None,
                s_down_t=None, b_up=0x3000, p1=0x4000, p2=0x5000, p_bias=0x6000)
    base.update(kw)
    return pb.pi_ffn_desc(**base)


def _create(lib, desc):
    h = C.c_void_p()
    rc = lib.pi_ffn_create(C.byref(desc), C.byref(h))
    if rc == 0:
        lib.pi_ffn_destroy(h)
    return rc


def test_create_validation(lib):
    assert _create(lib, _desc()) == pb.PI_OK
    assert _create(lib, _desc(d_model=0)) == pb.PI_ERR_INVALID_ARG
    assert _create(lib, _desc(act=7)) == pb.PI_ERR_INVALID_ARG
    assert _create(lib, _desc(wtype=9)) == pb.PI_ERR_INVALID_ARG
    assert _create(lib, _desc(b_up=None)) == pb.PI_ERR_INVALID_ARG           # ReLU needs b1
    assert _create(lib, _desc(act=pb.PI_ACT_SWIGLU)) == pb.PI_ERR_INVALID_ARG  # SwiGLU needs W_gate
    assert _create(lib, _desc(act=pb.PI_ACT_SWIGLU, w_gate=0x7000)) == pb.PI_OK
    assert _create(lib, _desc(wtype=pb.PI_W_INT4G32)) == pb.PI_ERR_INVALID_ARG  # scales missing
    assert _create(lib, _desc(wtype=pb.PI_W_INT4G32, s_up=0x8000, s_down_t=0x9000)) == pb.PI_OK
    assert _create(lib, _desc(wtype=pb.PI_W_INT4G32, s_up=0x8000, s_down_t=0x9000, d_model=48)) == \
        pb.PI_ERR_UNSUPPORTED                                                   # d % 32 for int4
    assert _create(lib, _desc(d_model=60)) == pb.PI_ERR_UNSUPPORTED             # d % 8
    assert _create(lib, _desc(rank=12)) == pb.PI_ERR_UNSUPPORTED                # fp16 rank % 8
    assert _create(lib, _desc(wtype=pb.PI_W_F32)) == pb.PI_ERR_UNSUPPORTED      # u/predictor type mismatch
    assert _create(lib, _desc(wtype=pb.PI_W_F32, ptype=pb.PI_W_F32)) == pb.PI_OK
    assert _create(lib, _desc(w_up=0x1008)) == pb.PI_ERR_MISALIGNED
    assert _create(lib, _desc(hot_prefix=200)) == pb.PI_ERR_INVALID_ARG
    assert _create(lib, _desc(d_model=32768)) == pb.PI_ERR_UNSUPPORTED


def test_entry_points_reject_bad_arguments_without_launching(lib):
    desc = _desc()
    h = C.c_void_p()
    assert lib.pi_ffn_create(C.byref(desc), C.byref(h)) == pb.PI_OK
    try:
        vp = C.c_void_p
        ws = vp(0x10000)
        # null handle / pointers
        assert lib.pi_predict(None, vp(0x100), 1, vp(0x200), vp(0x300), ws, 1 << 20, None) == pb.PI_ERR_INVALID_ARG
        assert lib.pi_predict(h, None, 1, vp(0x200), vp(0x300), ws, 1 << 20, None) == pb.PI_ERR_INVALID_ARG
        # batch out of range
        assert lib.pi_predict(h, vp(0x100), 33, vp(0x200), vp(0x300), ws, 1 << 20, None) == pb.PI_ERR_UNSUPPORTED
        assert lib.pi_predict(h, vp(0x100), -1, vp(0x200), vp(0x300), ws, 1 << 20, None) == pb.PI_ERR_UNSUPPORTED
        # misaligned
        assert lib.pi_predict(h, vp(0x104), 1, vp(0x200), vp(0x300), ws, 1 << 20, None) == pb.PI_ERR_MISALIGNED
        # missing workspace
        assert lib.pi_predict(h, vp(0x100), 1, vp(0x200), vp(0x300), None, 0, None) == pb.PI_ERR_WORKSPACE
        # unknown flag bits
        assert lib.pi_sparse_ffn(h, vp(0x100), 1, vp(0x200), vp(0x300), vp(0x400), 64, ws, 1 << 20, None) == \
            pb.PI_ERR_INVALID_ARG
        # batch 0 is a no-op
        assert lib.pi_decode_ffn(h, vp(0x100), 0, vp(0x400), None, None, 0, ws, 1 << 20, None) == pb.PI_OK
        # stacks: no fp32 layers, no ACCUMULATE flag
        arr = (vp * 1)(h)
        assert lib.pi_decode_ffn_stack(arr, 1, vp(0x100), 1, None, None, 1, ws, 1 << 20, None) == \
            pb.PI_ERR_INVALID_ARG
        assert lib.pi_decode_ffn_stack(arr, 0, vp(0x100), 1, None, None, 0, ws, 1 << 20, None) == \
            pb.PI_ERR_INVALID_ARG
        assert lib.pi_workspace_size(None, 1, 1, C.byref(C.c_size_t())) == pb.PI_ERR_INVALID_ARG
        assert lib.pi_workspace_size(arr, 1, 64, C.byref(C.c_size_t())) == pb.PI_ERR_UNSUPPORTED
    finally:
        lib.pi_ffn_destroy(h)


def test_static_entry_and_status_calls_check_arguments_first(lib):
    """pi_decode_ffn_static, pi_workspace_init and pi_get_device_status
    reject bad arguments before any CUDA call (none is made on this host)."""
    desc = _desc()
    h = C.c_void_p()
    assert lib.pi_ffn_create(C.byref(desc), C.byref(h)) == pb.PI_OK
    try:
        vp = C.c_void_p
        st = lib.pi_decode_ffn_static
        assert st(None, vp(0x100), vp(0x200), None, None, 0, None, None) == pb.PI_ERR_INVALID_ARG
        assert st(h, None, vp(0x200), None, None, 0, None, None) == pb.PI_ERR_INVALID_ARG
        assert st(h, vp(0x100), None, None, None, 0, None, None) == pb.PI_ERR_INVALID_ARG
        assert st(h, vp(0x104), vp(0x200), None, None, 0, None, None) == pb.PI_ERR_MISALIGNED
        assert st(h, vp(0x100), vp(0x208), None, None, 0, None, None) == pb.PI_ERR_MISALIGNED
        assert st(h, vp(0x100), vp(0x200), vp(0x308), None, 0, None, None) == pb.PI_ERR_MISALIGNED
        assert st(h, vp(0x100), vp(0x200), None, vp(0x404), 0, None, None) == pb.PI_ERR_MISALIGNED
        assert st(h, vp(0x100), vp(0x200), None, None, 0, vp(0x502), None) == pb.PI_ERR_MISALIGNED
        assert st(h, vp(0x100), vp(0x200), None, None, 8, None, None) == pb.PI_ERR_INVALID_ARG
        assert lib.pi_workspace_init(None, 1024, None) == pb.PI_ERR_INVALID_ARG
        assert lib.pi_workspace_init(vp(0x100), 0, None) == pb.PI_ERR_INVALID_ARG
        assert lib.pi_get_device_status(None, None, C.byref(C.c_int())) == pb.PI_ERR_INVALID_ARG
        assert lib.pi_get_device_status(vp(0x100), None, None) == pb.PI_ERR_INVALID_ARG
    finally:
        lib.pi_ffn_destroy(h)


def test_wait_fault_hook_validation(lib):
    """The failure-reporting test hook rejects a CTA index below -1 and a
    withheld slice without a wait limit; (-1, 0) restores normal runs."""
    assert lib.pi_debug_wait_fault(-2, 0) == pb.PI_ERR_INVALID_ARG
    assert lib.pi_debug_wait_fault(0, 0) == pb.PI_ERR_INVALID_ARG
    assert lib.pi_debug_wait_fault(-1, 0) == pb.PI_OK
