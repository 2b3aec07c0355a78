"""pi_decode_ffn_static: the batch-1 decode step on the library's static
device scratch, for callers that cannot allocate device memory at decode
time (a plugin in a runtime that hands out no device memory, an engine whose
caching allocator already holds all of HBM, a loop that cannot afford
cudaMalloc's implicit synchronisation).

Each case runs two consecutive calls of the static entry point and of the
workspace entry point pi_decode_ffn on the same layer and tokens.  Both run
the same kernels in the same arithmetic order, so the active sets, counts
and y must be identical bit for bit; y is also checked against the CPU
oracle's masked sum over the GPU's sets (outside the rounding band the sets
must be the oracle's), and the device status must be PI_OK.  The cases cover
the fused fp16 and int4 kernels and the multi-kernel fp32 path.  A last check
makes more static calls after the set-up and asserts that the device's free
memory and torch's allocation did not move.  This file is collected last so
that it also runs after every other GPU test in the same process; it passes
alone in a fresh process as well (the first call does the per-device set-up).
"""
import os
import re

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import inputs
from parity import assert_outputs, compare_sets, gpu_sets, host_layer

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pi_ffn.h")

CASES = [
    ("opt7b_f16", dict(d=512, f=2085, r=128)),            # fused fp16 ReLU kernel, ragged last mask word
    ("opt7b_f16", dict(d=4096, f=4096, r=256)),           # fused fp16, d = 4096
    ("llama70b_swiglu_int4", dict(d=512, f=1000, r=64)),  # fused int4 SwiGLU kernel
    ("opt_tiny_f32", dict(d=256, f=1000, r=32)),          # fp32 layer: predictor + gather + reduce kernels
]


def test_header_scratch_size_matches_binding():
    text = open(HEADER).read()
    m = re.search(r"#define PI_STATIC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m, "PI_STATIC_SCRATCH_BYTES not found in the header"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == pb.PI_STATIC_SCRATCH_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", CASES, ids=[f"{n}-d{k['d']}-f{k['f']}" for n, k in CASES])
def test_static_entry_matches_workspace_entry(cuda_device, name, kw):
    dev = cuda_device
    cfg = inputs.CONFIGS[name].scaled(**kw)
    lt = inputs.make_layer(cfg, 0, seed=23)
    L = host_layer(lt)
    layer = pb.FfnLayer.from_tensors(lt.to(dev))
    assert pb.pi_workspace_size([layer], 1) <= pb.PI_STATIC_SCRATCH_BYTES
    ws = pb.make_workspace([layer], 1, dev)
    toks = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 2, seed=29))
    # small, so that its fp32 rounding stays far below the tolerance of the delta
    y0 = 1e-3 * torch.randn((1, cfg.d), generator=torch.Generator().manual_seed(31))
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    for call in range(2):
        flags = 0 if call == 0 else pb.PI_FFN_ACCUMULATE  # the second call accumulates into a non-zero y
        u_host = toks[call:call + 1].contiguous()
        u = u_host.to(dev)
        y_ref, y = y0.to(dev), y0.to(dev)
        idx_ref = torch.full((1, cfg.f), -7, dtype=torch.int32, device=dev)
        idx = idx_ref.clone()
        cnt_ref = torch.full((1,), -7, dtype=torch.int32, device=dev)
        cnt = cnt_ref.clone()
        pb.pi_decode_ffn(layer, u, y_ref, ws, idx=idx_ref, count=cnt_ref, flags=flags)
        pb.pi_decode_ffn_static(layer, u, y, idx=idx, count=cnt, flags=flags, dev_status=status)
        torch.cuda.synchronize()
        assert pb.pi_get_device_status(ws) == 0
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        c = int(cnt_ref.item())
        assert int(cnt.item()) == c, f"call {call}: counts {int(cnt.item())} vs {c}"
        assert torch.equal(idx[0, :c], idx_ref[0, :c]), f"call {call}: active sets differ"
        assert torch.equal(y, y_ref), f"call {call}: y differs from pi_decode_ffn's"
        # against the oracle: the sets outside the rounding band, and y over the GPU's set
        pr = oracle.predict(L, u_host.numpy())
        sets, _, _ = compare_sets(gpu_sets(idx, cnt), pr, cfg.f)
        delta = oracle.ffn_masked(L, u_host.numpy(), sets)
        got = (y.cpu().double() - (y0.double() if call else 0.0)).numpy()
        assert_outputs(got, delta, cfg.wtype, f"static call {call}")


@pytest.mark.gpu
def test_static_entry_allocates_nothing(cuda_device):
    """After the first call (the set-up), further static calls change neither
    the device's free memory nor torch's allocation."""
    dev = cuda_device
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=512, f=2085, r=128)
    layer = pb.FfnLayer.from_tensors(inputs.make_layer(cfg, 0, seed=43).to(dev))
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 1, seed=47)).to(dev)
    y = torch.empty((1, cfg.d), device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    pb.pi_decode_ffn_static(layer, u, y, dev_status=status)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    alloc0 = torch.cuda.memory_allocated(dev)
    for _ in range(3):
        pb.pi_decode_ffn_static(layer, u, y, dev_status=status)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert free1 == free0, f"device free memory moved by {free0 - free1} bytes"
    assert torch.cuda.memory_allocated(dev) == alloc0
    assert int(status.item()) == 0


@pytest.mark.gpu
def test_static_entry_rejects_layer_beyond_scratch(cuda_device):
    """A layer whose batch-1 scratch exceeds the static array is refused on the
    host before anything is launched; y is left untouched.  The weights are
    allocated at full size, so the call would stay in bounds even if it ran."""
    dev = cuda_device
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=16384, f=64, r=16)
    lt = inputs.make_layer(cfg, 0, seed=37).to(dev)
    layer = pb.FfnLayer.from_tensors(lt)
    assert pb.pi_workspace_size([layer], 1) > pb.PI_STATIC_SCRATCH_BYTES
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 1, seed=41)).to(dev)
    y = torch.full((1, cfg.d), 3.0, device=dev)
    with pytest.raises(pb.PiError) as err:
        pb.pi_decode_ffn_static(layer, u, y)
    assert err.value.status == pb.PI_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(y == 3.0)
