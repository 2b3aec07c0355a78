"""Offline frequency profiling on the device: the calibration pass measures
firing counts with the library's own pi_predict on an OPT-7B-shaped layer
stored in seeded random order, stores the neurons hot-first, and the
reordered layer's decode step must still match the CPU oracle.

The generator's firing probabilities are never shown to the calibration; the
test uses them only to check the recovered order.  The generator caps the
207 most popular neurons at p = 0.99 and the neuron of popularity rank 256
sits at p ~ 0.84, so over 512 calibration tokens the measured top 64 must lie
in the generator's top 256.
"""
import numpy as np
import pytest
import torch

from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import calibrate, inputs
from parity import Gpu, check_layer

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_calibrate_with_pi_predict_then_decode_matches_oracle(cuda_device):
    dev = cuda_device
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(sort_neurons=False)
    lt = inputs.make_layer(cfg, 0, seed=61, device=dev)
    assert lt.hot_prefix == 0
    layer = pb.FfnLayer.from_tensors(lt)
    B = 8
    ws = pb.make_workspace([layer], B, dev)

    def predict(u):
        idx = torch.empty((u.shape[0], cfg.f), dtype=torch.int32, device=dev)
        cnt = torch.empty((u.shape[0],), dtype=torch.int32, device=dev)
        pb.pi_predict(layer, u, idx, cnt, ws)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        return [idx[b, :cnt[b]] for b in range(len(cnt))]

    batches = [inputs.layer_input(cfg, inputs.make_tokens(cfg, step, B, seed=67)).to(dev) for step in range(64)]
    lr, cal = calibrate.calibrate_layer(lt, predict, batches, frac=0.2)
    assert pb.pi_get_device_status(ws) == 0
    assert cal.tokens == 512
    assert np.all(np.diff(cal.counts) <= 0)
    assert cal.hot_prefix == calibrate.hot_prefix_fraction(cfg.f, 0.2)
    true_top = set(np.argsort(-lt.p, kind="stable")[:256].tolist())
    assert all(i in true_top for i in cal.perm[:64].tolist())
    # the measured mean firing rate of the prefix estimates the generator's
    assert cal.hot_p_mean == pytest.approx(float(lt.p[cal.perm[:cal.hot_prefix]].mean()), rel=0.1)
    # the reordered layer, through the library at batch 1 (fused kernel) and 4
    del layer, ws
    g = Gpu(lr.to("cpu"), 4)
    for B_chk in (1, 4):
        u = inputs.layer_input(cfg, inputs.make_tokens(cfg, 100, B_chk, seed=71))
        check_layer(lr.to("cpu"), u, g)


def test_size_rank_on_the_device(cuda_device):
    """Predictor sizing with the library's own calls: each truncated predictor
    through pi_predict, the FFN output over its sets through pi_sparse_ffn,
    against the full rank-1024 predictor's sets on an OPT-7B-shaped layer.
    The full rank reproduces the reference exactly (shift 0, recall 1), the
    shift falls as the rank grows, and the choice is the smallest candidate
    within the 0.4% cosine shift."""
    dev = cuda_device
    cfg = inputs.CONFIGS["opt7b_f16"]
    lt = inputs.make_layer(cfg, 0, seed=73, device=dev)
    ranks = (256, 512, 1024)
    cut = {r: calibrate.truncate_predictor(lt, r) for r in ranks}
    layers = {r: pb.FfnLayer.from_tensors(cut[r]) for r in ranks}
    B = 8
    ws = pb.make_workspace(list(layers.values()), B, dev)

    def predict_at(r, u):
        idx = torch.empty((u.shape[0], cfg.f), dtype=torch.int32, device=dev)
        cnt = torch.empty((u.shape[0],), dtype=torch.int32, device=dev)
        pb.pi_predict(layers[r], u, idx, cnt, ws)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        return [idx[b, :cnt[b]] for b in range(len(cnt))]

    def ffn(u, sets):
        idx = torch.zeros((u.shape[0], cfg.f), dtype=torch.int32)
        cnt = torch.zeros((u.shape[0],), dtype=torch.int32)
        for b, s in enumerate(sets):
            idx[b, :len(s)] = torch.from_numpy(np.asarray(s, np.int32))
            cnt[b] = len(s)
        y = torch.empty((u.shape[0], cfg.d), device=dev)
        pb.pi_sparse_ffn(layers[1024], u, idx.to(dev), cnt.to(dev), y, ws)
        return y.cpu().numpy()

    batches = [inputs.layer_input(cfg, inputs.make_tokens(cfg, step, B, seed=79)).to(dev) for step in range(2)]
    ch = calibrate.size_rank(ranks, predict_at, ffn, lambda u: predict_at(1024, u), batches)
    assert pb.pi_get_device_status(ws) == 0
    full = ch.table[-1]
    assert full["rank"] == 1024 and full["mean_shift"] <= 1e-12 and full["recall"] == 1.0
    shifts = [row["mean_shift"] for row in ch.table]
    assert shifts[0] >= shifts[1] >= shifts[2]
    assert ch.met and ch.rank == min(row["rank"] for row in ch.table if row["mean_shift"] <= 0.004)
    print("rank sizing table:", ch.table)
