"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Sizes span several 32-neuron mask words, several CTA chunks of the gather
kernel and a ragged tail (f not a multiple of 32, B not a power of two).
Full-size single layers of every workload shape are checked element by
element on a few seeded tokens.
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


def small_cfg(name, **kw):
    return inputs.CONFIGS[name].scaled(**{**SMALL, **kw})


# ------------------------------------------------------------------ exact arithmetic

@pytest.mark.parametrize("act,wtype", [("relu", "f32"), ("relu", "f16"), ("relu", "int4g32")])
@pytest.mark.parametrize("B", [1, 3, 8])
def test_exact_arithmetic_bitwise(cuda_device, act, wtype, B):
    """Small-integer weights and inputs make every sum exact in fp32, so the
    active sets (ties s == 0 included) and y must match the oracle bitwise."""
    lt = inputs.make_exact_layer(d=256, f=1000, r=64, act=act, wtype=wtype, seed=B)
    g = Gpu(lt, 8)
    u = inputs.make_exact_tokens(256, B, seed=B, dtype=torch.float32 if wtype == "f32" else torch.float16)
    L = host_layer(lt)
    pr = oracle.predict(L, u.numpy())
    idx, cnt = g.predict(u.cuda())
    for b, s in enumerate(gpu_sets(idx, cnt)):
        assert np.array_equal(s, pr["idx"][b])
    y_ref = oracle.ffn_masked(L, u.numpy(), pr["idx"])
    y = g.sparse_ffn(u.cuda(), pr["idx"]).cpu().numpy()
    assert np.array_equal(y.astype(np.float64), y_ref)
    yd, idx2, cnt2 = g.decode(u.cuda())
    assert np.array_equal(yd.cpu().numpy().astype(np.float64), y_ref)
    for b, s in enumerate(gpu_sets(idx2, cnt2)):
        assert np.array_equal(s, pr["idx"][b])


def test_exact_ties_do_not_fire(cuda_device):
    """fires iff s > 0: shift the bias of some neurons so that their (exact)
    score is exactly 0; neither side may select them, and the rest of the set
    is unchanged."""
    lt = inputs.make_exact_layer(d=256, f=640, r=64, act="relu", wtype="f16", seed=5)
    u = inputs.make_exact_tokens(256, 1, seed=5)
    L = host_layer(lt)
    s = oracle.predict(L, u.numpy())["s"][0]
    tie = np.arange(0, 640, 7)
    b = lt.p_bias.clone()
    b[tie] -= torch.from_numpy(s[tie]).float()
    lt2 = inputs.LayerTensors(**{**lt.__dict__, "p_bias": b, "b_up": b})
    pr = oracle.predict(host_layer(lt2), u.numpy())
    assert np.all(pr["s"][0][tie] == 0)
    g = Gpu(lt2, 1)
    idx, cnt = g.predict(u.cuda())
    got = gpu_sets(idx, cnt)[0]
    assert np.array_equal(got, pr["idx"][0]) and not np.any(np.isin(tie, got))


# ------------------------------------------------------------------ seeded workloads, small

@pytest.mark.parametrize("name", inputs.CONFIG_ORDER)
@pytest.mark.parametrize("B", [1, 3, 8])
def test_layer_parity_small(cuda_device, name, B):
    cfg = small_cfg(name) if name != "opt_tiny_f32" else inputs.CONFIGS[name].scaled(f=1061)
    lt = inputs.make_layer(cfg, layer=1, seed=7)
    g = Gpu(lt, 8)
    for step in range(2):
        x = inputs.make_tokens(cfg, step, B, seed=7)
        rep = check_layer(lt, inputs.layer_input(cfg, x), g)
        assert rep["band_frac"] < 0.01


@pytest.mark.parametrize("name", ["opt7b_f16", "llama70b_swiglu_int4"])
def test_hot_dense_and_index_modes_agree(cuda_device, name):
    """Reading the hot prefix densely changes bytes, never results."""
    cfg = small_cfg(name)
    lt = inputs.make_layer(cfg, 0, seed=3)
    g = Gpu(lt, 8)
    x = inputs.make_tokens(cfg, 0, 4, seed=3)
    u = inputs.layer_input(cfg, x)
    rep_d = check_layer(lt, u, g, flags=pb.PI_FFN_HOT_DENSE)
    rep_i = check_layer(lt, u, g, flags=pb.PI_FFN_HOT_INDEX)
    yd, _, _ = g.decode(u.cuda(), flags=pb.PI_FFN_HOT_DENSE)
    yi, _, _ = g.decode(u.cuda(), flags=pb.PI_FFN_HOT_INDEX)
    den = yi.abs().max()
    assert float((yd - yi).abs().max() / den) < 1e-6


def test_determinism_bitwise(cuda_device):
    cfg = small_cfg("opt7b_f16")
    lt = inputs.make_layer(cfg, 0, seed=4)
    g = Gpu(lt, 8)
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 8, seed=4)).cuda()
    a = g.decode(u)
    b = g.decode(u)
    for t1, t2 in zip(a, b):
        assert torch.equal(t1, t2)


# ------------------------------------------------------------------ edge cases

@pytest.fixture(scope="module")
def relu_small():
    cfg = small_cfg("opt7b_f16")
    lt = inputs.make_layer(cfg, 0, seed=11)
    return cfg, lt, Gpu(lt, 8)


def test_empty_sets_give_exact_zero(cuda_device, relu_small):
    cfg, lt, g = relu_small
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 3, seed=11)).cuda()
    y = g.sparse_ffn(u, [np.array([], np.int32)] * 3)
    assert torch.all(y == 0) and not torch.any(torch.signbit(y))


def test_all_true_mask_equals_dense(cuda_device, relu_small):
    cfg, lt, g = relu_small
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 1, 2, seed=11))
    L = host_layer(lt)
    y = g.sparse_ffn(u.cuda(), [np.arange(cfg.f, dtype=np.int32)] * 2).cpu().numpy()
    assert_outputs(y, oracle.ffn_dense(L, u.numpy()), cfg.wtype)


def test_single_neuron_sets(cuda_device, relu_small):
    cfg, lt, g = relu_small
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 2, 1, seed=11))
    L = host_layer(lt)
    pre = oracle.relu_preact(L, u.numpy())[0]
    for i in (0, 31, 32, int(np.argmax(pre)), cfg.f - 1):
        y = g.sparse_ffn(u.cuda(), [np.array([i], np.int32)]).cpu().numpy()
        y_ref = max(pre[i], 0.0) * lt.w_down_t[i].double().numpy()
        assert_outputs(y, y_ref[None, :], cfg.wtype, f"neuron {i}")


def test_lists_are_sets_and_bad_ids_flag_status(cuda_device, relu_small):
    cfg, lt, g = relu_small
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 3, 2, seed=11))
    L = host_layer(lt)
    S = [np.array([5, 900, 77, 5, 2084], np.int32), np.array([3, 1, 2], np.int32)]
    y = g.sparse_ffn(u.cuda(), S).cpu().numpy()
    assert g.status() == 0
    y_ref = oracle.ffn_masked(L, u.numpy(), [np.unique(s) for s in S])
    assert_outputs(y, y_ref, cfg.wtype)
    # an id >= f is skipped and reported through the device status word
    y = g.sparse_ffn(u.cuda(), [np.array([5, 900, 99999], np.int32), np.array([1, -4], np.int32)]).cpu().numpy()
    assert g.status() == pb.PI_ERR_DEVICE_STATUS
    assert g.status() == 0  # reading clears it
    y_ref = oracle.ffn_masked(L, u.numpy(), [np.array([5, 900], np.int32), np.array([1], np.int32)])
    assert_outputs(y, y_ref, cfg.wtype)


def test_accumulate_flag(cuda_device, relu_small):
    cfg, lt, g = relu_small
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 4, 2, seed=11)).cuda()
    S = [np.array([1, 2, 3], np.int32), np.array([10, 2000], np.int32)]
    y1 = g.sparse_ffn(u, S)
    y = torch.ones_like(y1)
    idx = torch.zeros((2, cfg.f), dtype=torch.int32)
    cnt = torch.tensor([3, 2], dtype=torch.int32)
    idx[0, :3] = torch.tensor([1, 2, 3]); idx[1, :2] = torch.tensor([10, 2000])
    pb.pi_sparse_ffn(g.layer, u, idx.cuda(), cnt.cuda(), y, g.ws, flags=pb.PI_FFN_ACCUMULATE)
    assert torch.equal(y, 1.0 + y1)


def test_literal_bias_norm_near_empty_sets(cuda_device):
    """The small fp32 layer with the literal sigma_i = ||W1_i|| bias predicts
    almost nothing: many tokens have empty sets and y must be exactly 0."""
    cfg = inputs.CONFIGS["opt_tiny_f32"].scaled(bias_norm="w1")
    lt = inputs.make_layer(cfg, 0, seed=0)
    g = Gpu(lt, 8)
    empties = 0
    for step in range(6):
        u = inputs.layer_input(cfg, inputs.make_tokens(cfg, step, 8, seed=0))
        rep = check_layer(lt, u, g)
        empties += sum(c == 0 for c in rep["count"])
    assert empties > 0


# ------------------------------------------------------------------ full-size single layers

@pytest.mark.slow
@pytest.mark.parametrize("name", inputs.CONFIG_ORDER)
def test_full_size_layer(cuda_device, name):
    """One full-size layer of each workload shape, element-by-element against
    the oracle on seeded tokens at the shape's batch sizes (<= 8 here)."""
    cfg = inputs.CONFIGS[name]
    lt = inputs.make_layer(cfg, layer=cfg.n_layers - 1, seed=0, device="cuda").to("cpu")
    g = Gpu(lt, 8)
    for B in [b for b in cfg.batches if b <= 8]:
        x = inputs.make_tokens(cfg, 0, B, seed=0)
        check_layer(lt, inputs.layer_input(cfg, x), g)


@pytest.mark.parametrize("name,B", [("llama13b_swiglu_f16", 1), ("llama13b_swiglu_f16", 4), ("opt7b_f16", 1),
                                    ("opt7b_f16", 8)])
def test_repeated_decode_is_bitwise_stable(cuda_device, name, B):
    """A full-size layer decoded 200 times on the same tokens gives the same
    bits every time: sums run in a fixed order, so any difference is a race
    (a partial read before it is written, a buffer reused too early)."""
    cfg = inputs.CONFIGS[name]
    lt = inputs.make_layer(cfg, layer=cfg.n_layers - 1, seed=0, device="cuda")
    g = Gpu(lt, 8)
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, B, seed=0).cuda()).cuda()
    y0 = g.decode(u)[0].clone()
    bad = sum(int(not torch.equal(g.decode(u)[0], y0)) for _ in range(200))
    assert bad == 0, f"{bad} of 200 repeated decodes differ"
    assert g.status() == 0


@pytest.mark.parametrize("start", [0, 1000003])
def test_reduction_slices_whatever_the_arrival_counter_holds(cuda_device, start):
    """Batch 1: the CTAs that finish their stream first sum the slices of y,
    by their arrival ticket mod the grid size.  From any counter value that
    is a permutation of the slices, so y is bitwise the same; the counter
    is back at its start value after every launch."""
    cfg = inputs.CONFIGS["opt7b_f16"]
    lt = inputs.make_layer(cfg, layer=cfg.n_layers - 1, seed=0, device="cuda")
    g = Gpu(lt, 1)
    u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 1, seed=0).cuda()).cuda()
    y0 = g.decode(u)[0].clone()  # with the id lists: every CTA stays to the end
    ticket = g.ws[68:72].view(torch.int32)  # the arrival counter's word in the workspace header
    assert int(ticket.item()) == 0
    ticket.fill_(start)
    y = torch.empty(1, lt.d, device="cuda")
    for k in range(50):  # without id lists: the CTAs past the last slice leave early
        y.fill_(float("nan"))
        pb.pi_decode_ffn(g.layer, u, y, g.ws)
        assert torch.equal(y, y0), f"launch {k} differs"
    torch.cuda.synchronize()
    assert int(ticket.item()) == start
    assert g.status() == 0


# ------------------------------------------------------------------ every batch size of each path

@pytest.mark.parametrize("name,batches", [
    ("opt7b_f16", list(range(2, 17))),             # batch kernels 2..8, tcgen05 9..16
    ("llama13b_swiglu_f16", [2, 5, 7, 8, 9, 12]),
    ("llama70b_swiglu_int4", [2, 3, 5, 6]),        # tcgen05 from 2 tokens (int4)
])
def test_every_batch_size_matches_the_oracle(cuda_device, name, batches):
    """Predictor, sparse FFN and decode step against the oracle at each batch
    size, across the boundaries where the library changes kernels (the fp16
    batch kernels end at 8 tokens, the tensor-core path starts at 9 for fp16
    and at 2 for int4)."""
    cfg = small_cfg(name, d=1024 if name != "llama70b_swiglu_int4" else 512)
    lt = inputs.make_layer(cfg, 0, seed=83)
    g = Gpu(lt, 16)
    for B in batches:
        u = inputs.layer_input(cfg, inputs.make_tokens(cfg, B, B, seed=89))
        check_layer(lt, u, g)


def test_batch_on_a_width_the_batch_kernels_do_not_take(cuda_device):
    """d = 520 is not a multiple of 64: batches 2..8 run on the CUDA-core
    multi-kernel path, which must match the oracle as well."""
    cfg = small_cfg("opt7b_f16", d=520)
    lt = inputs.make_layer(cfg, 0, seed=97)
    g = Gpu(lt, 8)
    for B in (2, 5, 8):
        u = inputs.layer_input(cfg, inputs.make_tokens(cfg, B, B, seed=101))
        check_layer(lt, u, g)
