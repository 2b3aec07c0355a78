"""pi_decode_ffn_static: the batch-1 decode step on the library's static
device scratch, for callers that cannot allocate device memory.

Each case runs two consecutive calls of the static entry point and of the
workspace entry point pi_decode_ffn on the same layer and tokens and compares
them: identical active sets and counts, y within the parity tolerance of the
weight type, device status PI_OK.  The cases cover the fused fp16 and int4
kernels and the multi-kernel fp32 path.  This file is collected last so that
it also runs after every other GPU test in the same process; it passes alone
in a fresh process as well (the first call does the per-device set-up).
"""
import os
import re

import numpy as np
import pytest
import torch

from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import inputs

TOL = {"f32": 1e-5, "f16": 2e-3, "int4g32": 2e-3}
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pi_ffn.h")

CASES = [
    ("opt7b_f16", dict(d=512, f=2085, r=128)),            # fused fp16 ReLU kernel, ragged last mask word
    ("opt7b_f16", dict(d=4096, f=4096, r=256)),           # fused fp16, d = 4096: the largest partial rows
    ("llama70b_swiglu_int4", dict(d=512, f=1000, r=64)),  # fused int4 SwiGLU kernel
    ("opt_tiny_f32", dict(d=256, f=1000, r=32)),          # fp32 layer: predictor + gather + reduce kernels
]


def test_header_scratch_size_matches_binding():
    text = open(HEADER).read()
    m = re.search(r"#define PI_STATIC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", text)
    assert m, "PI_STATIC_SCRATCH_BYTES not found in the header"
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == pb.PI_STATIC_SCRATCH_BYTES


def _rel_err(a: np.ndarray, b: np.ndarray) -> float:
    den = np.max(np.abs(b))
    num = np.max(np.abs(a.astype(np.float64) - b.astype(np.float64)))
    return (0.0 if num == 0 else np.inf) if den == 0 else num / den


@pytest.mark.gpu
@pytest.mark.parametrize("name,kw", CASES, ids=[f"{n}-d{k['d']}-f{k['f']}" for n, k in CASES])
def test_static_entry_matches_workspace_entry(cuda_device, name, kw):
    dev = cuda_device
    cfg = inputs.CONFIGS[name].scaled(**kw)
    lt = inputs.make_layer(cfg, 0, seed=23).to(dev)
    layer = pb.FfnLayer.from_tensors(lt)
    assert pb.pi_workspace_size([layer], 1) <= pb.PI_STATIC_SCRATCH_BYTES
    ws = pb.make_workspace([layer], 1, dev)
    toks = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 2, seed=29)).to(dev)
    y0 = torch.randn((1, cfg.d), generator=torch.Generator().manual_seed(31)).to(dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    for call in range(2):
        # the second call accumulates into a non-zero y
        flags = 0 if call == 0 else pb.PI_FFN_ACCUMULATE
        u = toks[call:call + 1].contiguous()
        y_ref, y = y0.clone(), y0.clone()
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
        e = _rel_err(y.cpu().numpy(), y_ref.cpu().numpy())
        assert e <= TOL[cfg.wtype], f"call {call}: rel err {e:.3e} > {TOL[cfg.wtype]}"


@pytest.mark.gpu
def test_static_entry_rejects_layer_beyond_scratch(cuda_device):
    """A layer whose batch-1 scratch exceeds the static array is refused on the
    host before anything is launched; y is left untouched.  The weights are
    allocated at full size, so the call would stay in bounds even if it ran."""
    dev = cuda_device
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=8192, f=64, r=8)
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
