"""GPU parity of the tensor-core (tcgen05) path, taken at batches 16..32.

At these batches pi_predict, pi_sparse_ffn, pi_decode_ffn and the stack run
the predictor GEMMs, the gathered up/gate GEMM and the down GEMM on tensor
cores (tokens padded to 32 MMA columns, stream-K over all SMs).  Sizes span
several 128-row tiles with a ragged last tile (f not a multiple of 32 or 128),
several K steps with a ragged last step (d or r not a multiple of 128) and
batches that are not a power of two.
"""
import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import inputs
from parity import Gpu, assert_outputs, check_layer, compare_sets, gpu_sets, host_layer

pytestmark = pytest.mark.gpu

SMALL = dict(d=512, f=2085, r=128)


@pytest.mark.parametrize("wtype", ["f16", "int4g32"])
@pytest.mark.parametrize("B", [16, 32])
def test_exact_arithmetic_tc(cuda_device, wtype, B):
    """Small-integer weights and inputs: every predictor sum is exact, so the
    active sets (ties included) match the oracle bitwise; fp16 outputs are
    exact too.  For int4 the fp16 rounding of the activation before the down
    GEMM may round a few large activations, so y is checked to 1e-3."""
    lt = inputs.make_exact_layer(d=256, f=1000, r=64, act="relu", wtype=wtype, seed=40 + B)
    g = Gpu(lt, 32)
    u = inputs.make_exact_tokens(256, B, seed=B)
    L = host_layer(lt)
    pr = oracle.predict(L, u.numpy())
    idx, cnt = g.predict(u.cuda())
    for b, s in enumerate(gpu_sets(idx, cnt)):
        assert np.array_equal(s, pr["idx"][b]), f"token {b}"
    y = g.sparse_ffn(u.cuda(), pr["idx"]).cpu().numpy()
    y_ref = oracle.ffn_masked(L, u.numpy(), pr["idx"])
    yd, idx2, cnt2 = g.decode(u.cuda())
    for b, s in enumerate(gpu_sets(idx2, cnt2)):
        assert np.array_equal(s, pr["idx"][b]), f"decode token {b}"
    if wtype == "f16":
        assert np.array_equal(y.astype(np.float64), y_ref)
        assert np.array_equal(yd.cpu().numpy().astype(np.float64), y_ref)
    else:
        for yy in (y, yd.cpu().numpy()):
            den = np.abs(y_ref).max()
            assert np.abs(yy - y_ref).max() <= 1e-3 * den
    assert g.status() == 0


CASES = {
    "relu_f16": ("opt7b_f16", SMALL),
    "relu_f16_ragged": ("opt7b_f16", dict(d=520, f=700, r=72)),
    "swiglu_f16": ("llama13b_swiglu_f16", SMALL),
    "swiglu_int4": ("llama70b_swiglu_int4", SMALL),
    "relu_int4": ("llama70b_swiglu_int4", dict(SMALL, act="relu", mean_p=0.1)),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("B", [16, 17, 32])
def test_layer_parity_tc(cuda_device, case, B):
    name, kw = CASES[case]
    cfg = inputs.CONFIGS[name].scaled(**kw)
    lt = inputs.make_layer(cfg, layer=2, seed=17)
    g = Gpu(lt, 32)
    for step in range(2):
        x = inputs.make_tokens(cfg, step, B, seed=17)
        rep = check_layer(lt, inputs.layer_input(cfg, x), g)
        assert rep["band_frac"] < 0.01


def test_tc_empty_union_gives_zero(cuda_device):
    """Caller sets that are all empty: y = 0 exactly, and += leaves y as is."""
    cfg = inputs.CONFIGS["llama70b_swiglu_int4"].scaled(**SMALL)
    lt = inputs.make_layer(cfg, 0, seed=5)
    g = Gpu(lt, 32)
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 16, seed=5)).cuda()
    y = g.sparse_ffn(u, [np.array([], np.int32)] * 16)
    assert torch.all(y == 0)
    idx = torch.zeros((16, cfg.f), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(16, dtype=torch.int32, device="cuda")
    y0 = torch.randn(16, cfg.d, device="cuda")
    y1 = y0.clone()
    pb.pi_sparse_ffn(g.layer, u, idx, cnt, y1, g.ws, flags=pb.PI_FFN_ACCUMULATE)
    assert torch.equal(y0, y1)
    assert g.status() == 0


def test_tc_determinism_bitwise(cuda_device):
    cfg = inputs.CONFIGS["llama70b_swiglu_int4"].scaled(**SMALL)
    lt = inputs.make_layer(cfg, 0, seed=6)
    g = Gpu(lt, 32)
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 32, seed=6)).cuda()
    a = g.decode(u)
    b = g.decode(u)
    for t1, t2 in zip(a, b):
        assert torch.equal(t1, t2)


def test_tc_decode_without_id_lists(cuda_device):
    """pi_decode_ffn at B >= 16 without idx/count (the compaction is then
    skipped; the FFN kernels list their tiles from the mask words) gives the
    same y, bitwise, as the call that also returns the id lists."""
    cfg = inputs.CONFIGS["llama70b_swiglu_int4"].scaled(**SMALL)
    lt = inputs.make_layer(cfg, 0, seed=9)
    g = Gpu(lt, 32)
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 24, seed=9)).cuda()
    y1, _, _ = g.decode(u)
    y2 = torch.full_like(y1, float("nan"))
    pb.pi_decode_ffn(g.layer, u, y2, g.ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert g.status() == 0


def test_tc_stack_composes_layers(cuda_device):
    """pi_decode_ffn_stack over 3 layers at B=16 equals three one-layer stack
    calls bitwise, traces included (the layer loop adds nothing of its own;
    each layer's arithmetic is covered by the single-layer parity tests)."""
    cfg = inputs.CONFIGS["llama70b_swiglu_int4"].scaled(d=512, f=700, r=64, n_layers=3)
    lts = [inputs.make_layer(cfg, l, seed=8).to("cuda") for l in range(cfg.n_layers)]
    layers = [pb.FfnLayer.from_tensors(lt) for lt in lts]
    ws = pb.make_workspace(layers, 32)
    B = 16
    x0 = inputs.make_tokens(cfg, 0, B, seed=8).cuda()
    xs = x0.clone()
    idx = torch.full((3, B, cfg.f), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((3, B), -1, dtype=torch.int32, device="cuda")
    pb.pi_decode_ffn_stack(layers, xs, ws, idx_trace=idx, count_trace=cnt)
    xr = x0.clone()
    for l, L in enumerate(layers):
        i1 = torch.full((1, B, cfg.f), -1, dtype=torch.int32, device="cuda")
        c1 = torch.full((1, B), -1, dtype=torch.int32, device="cuda")
        pb.pi_decode_ffn_stack([L], xr, ws, idx_trace=i1, count_trace=c1)
        assert torch.equal(c1[0], cnt[l])
        for b in range(B):
            n = int(cnt[l, b])
            assert torch.equal(i1[0, b, :n], idx[l, b, :n])
    torch.cuda.synchronize()
    assert pb.pi_get_device_status(ws) == 0
    assert torch.equal(xs, xr)
    assert not torch.equal(xs, x0)


@pytest.mark.slow
@pytest.mark.parametrize("name,B", [("llama70b_swiglu_int4", 16), ("llama70b_swiglu_int4", 32),
                                    ("opt7b_f16", 16)])
def test_full_size_layer_tc(cuda_device, name, B):
    """Full-size layers at the tensor-core batches, element by element."""
    cfg = inputs.CONFIGS[name]
    lt = inputs.make_layer(cfg, layer=cfg.n_layers - 1, seed=0, device="cuda").to("cpu")
    g = Gpu(lt, 32)
    x = inputs.make_tokens(cfg, 0, B, seed=0)
    check_layer(lt, inputs.layer_input(cfg, x), g)
