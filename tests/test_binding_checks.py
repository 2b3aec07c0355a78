"""The binding's own argument checks, on CPU.  The C ABI sees only pointers;
the binding checks each tensor's dtype, size, contiguity and device before
it calls the library, and raises ValueError.  No CUDA call is made here: a
layer handle is created from host tensors (creation validates pointers and
shapes only), and every call below fails in the binding."""
import os

import pytest
import torch

from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import inputs


@pytest.fixture(scope="module")
def layer():
    if not os.environ.get("PI_FFN_LIB"):  # another build given: use it as is
        from activation_sparse_decode_gemv_b200 import build
        build.build()
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=256, f=320, r=32)
    lt = inputs.make_layer(cfg, 0, seed=1)
    return pb.FfnLayer.from_tensors(lt)


def _ok(layer, B=2):
    u = torch.zeros((B, layer.d), dtype=torch.float16)
    y = torch.zeros((B, layer.d), dtype=torch.float32)
    idx = torch.zeros((B, layer.f), dtype=torch.int32)
    cnt = torch.zeros((B,), dtype=torch.int32)
    ws = torch.zeros(1024, dtype=torch.uint8)
    return u, y, idx, cnt, ws


def _raises(fn, match):
    with pytest.raises(ValueError, match=match):
        fn()


def test_token_shape_and_dtype(layer):
    u, y, idx, cnt, ws = _ok(layer)
    _raises(lambda: pb.pi_decode_ffn(layer, u[0], y, ws), r"u: shape")
    _raises(lambda: pb.pi_decode_ffn(layer, u[:, :128], y, ws), r"u: shape")
    _raises(lambda: pb.pi_decode_ffn(layer, u.float(), y, ws), r"u: dtype")
    _raises(lambda: pb.pi_predict(layer, u.float(), idx, cnt, ws), r"u: dtype")


def test_output_and_index_buffers(layer):
    u, y, idx, cnt, ws = _ok(layer)
    _raises(lambda: pb.pi_decode_ffn(layer, u, y[:1], ws), r"y: .* elements")
    _raises(lambda: pb.pi_decode_ffn(layer, u, y.half(), ws), r"y: dtype")
    _raises(lambda: pb.pi_decode_ffn(layer, u, y, ws, idx=idx.long()), r"idx: dtype")
    _raises(lambda: pb.pi_predict(layer, u, idx[:, :10], cnt, ws), r"idx: .* elements")
    _raises(lambda: pb.pi_predict(layer, u, idx, cnt[:1], ws), r"count: .* elements")
    _raises(lambda: pb.pi_sparse_ffn(layer, u, idx, cnt, y.t(), ws), r"y: must be contiguous")


def test_host_tensors_are_rejected(layer):
    u, y, idx, cnt, ws = _ok(layer)
    _raises(lambda: pb.pi_decode_ffn(layer, u, y, ws), r"u: must be a CUDA tensor")
    _raises(lambda: pb.pi_sparse_ffn(layer, u, idx, cnt, y, ws), r"must be a CUDA tensor")


def test_static_entry_is_batch_one(layer):
    u, y, idx, cnt, ws = _ok(layer)
    _raises(lambda: pb.pi_decode_ffn_static(layer, u, y), r"batch 1")
    _raises(lambda: pb.pi_decode_ffn_static(layer, u[:1], y[:1], dev_status=torch.zeros(1, dtype=torch.int64)),
            r"dev_status: dtype")
    _raises(lambda: pb.pi_decode_ffn_static(layer, u[:1], y[:1]), r"u: must be a CUDA tensor")


def test_stack_arguments(layer):
    _, _, _, _, ws = _ok(layer)
    x = torch.zeros((2, layer.d), dtype=torch.float32)
    _raises(lambda: pb.pi_decode_ffn_stack([], x, ws), r"at least one layer")
    _raises(lambda: pb.pi_decode_ffn_stack([layer], x.half(), ws), r"x: dtype")
    _raises(lambda: pb.pi_decode_ffn_stack([layer, layer], x,
                                           ws, idx_trace=torch.zeros((1, 2, layer.f), dtype=torch.int32)),
            r"idx_trace: .* elements")
    _raises(lambda: pb.pi_decode_ffn_stack([layer], x, ws, count_trace=torch.zeros((1, 1), dtype=torch.int32)),
            r"count_trace: .* elements")
