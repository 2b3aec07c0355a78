"""Offline hot/cold reordering from measured firing frequencies (host logic).

The predictor used for calibration here is the oracle's; on a GPU the same
functions take the library's pi_predict (see the calibrate module).  Pins:

* reordering is a pure relabelling of neurons: predictor scores move with
  their rows bit for bit, predicted sets map through the permutation, and
  the FFN output is the same sum in another order;
* on a layer stored in seeded random order, the measured counts recover the
  generator's popularity order (statistically);
* the hot-prefix rules against closed-form cases.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from activation_sparse_decode_gemv_b200 import calibrate, inputs


def _host(lt):
    return oracle.Layer(**lt.host_arrays())


def _u(cfg, step, B, seed):
    return inputs.layer_input(cfg, inputs.make_tokens(cfg, step, B, seed=seed))


@pytest.mark.parametrize("name,kw", [
    ("opt7b_f16", dict(d=256, f=320, r=32)),
    ("llama70b_swiglu_int4", dict(d=256, f=288, r=32)),
])
def test_reorder_is_a_relabelling(name, kw):
    cfg = inputs.CONFIGS[name].scaled(**kw)
    lt = inputs.make_layer(cfg, 0, seed=3)
    perm = np.random.default_rng(7).permutation(cfg.f)
    lr = calibrate.reorder_layer(lt, perm, hot_prefix=64, hot_p_mean=0.5)
    assert lr.hot_prefix == 64 and lr.hot_p_mean == 0.5
    if lt.b_up is not None:
        assert torch.equal(lr.b_up, lr.p_bias)
    assert torch.equal(lr.p1, lt.p1)
    L, Lr = _host(lt), _host(lr)
    u = _u(cfg, 0, 6, 3).numpy()
    pr, prr = oracle.predict(L, u), oracle.predict(Lr, u)
    # each score is computed from its own row: bitwise equal after relabelling
    assert np.array_equal(prr["s"], pr["s"][:, perm])
    mapped = calibrate.map_sets(pr["idx"], perm)
    for a, b in zip(mapped, prr["idx"]):
        assert np.array_equal(a, b)
    y = oracle.ffn_masked(L, u, pr["idx"])
    yr = oracle.ffn_masked(Lr, u, prr["idx"])
    assert np.allclose(yr, y, rtol=1e-12, atol=1e-15 * np.abs(y).max())


def test_reorder_rejects_bad_arguments():
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=256, f=320, r=32)
    lt = inputs.make_layer(cfg, 0, seed=1)
    with pytest.raises(ValueError):
        calibrate.reorder_layer(lt, np.arange(cfg.f - 1))
    with pytest.raises(ValueError):
        calibrate.reorder_layer(lt, np.zeros(cfg.f, np.int64))
    with pytest.raises(ValueError):
        calibrate.reorder_layer(lt, np.arange(cfg.f), hot_prefix=33)


def test_calibration_recovers_popularity_order():
    """A power-law layer stored in random order: after calibration on 768
    seeded tokens the stored order follows the generator's firing
    probabilities (which the calibration never sees)."""
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=256, f=1024, r=64, sort_neurons=False)
    lt = inputs.make_layer(cfg, 0, seed=11)
    L = _host(lt)
    batches = [_u(cfg, step, 64, 11) for step in range(12)]

    def predict(u):
        return oracle.predict(L, u.numpy())["idx"]

    lr, cal = calibrate.calibrate_layer(lt, predict, batches, frac=0.2)
    assert cal.tokens == 768
    assert np.all(np.diff(cal.counts) <= 0)
    assert cal.hot_prefix == 192 and lr.hot_prefix == 192
    assert cal.hot_p_mean == pytest.approx(cal.counts[:192].mean() / 768)
    # the generator's probabilities in the new order
    p_new = lt.p[cal.perm]
    assert np.array_equal(p_new, lr.p)
    true_top = set(np.argsort(-lt.p, kind="stable")[:128].tolist())
    meas_top = cal.perm[:64].tolist()
    assert sum(i in true_top for i in meas_top) >= 60
    # rank correlation over the neurons that fire often enough to be ranked
    sel = lt.p[cal.perm] >= 0.05
    rp = np.argsort(np.argsort(-p_new[sel]))
    rc = np.argsort(np.argsort(-cal.counts[sel].astype(float)))
    rho = np.corrcoef(rp, rc)[0, 1]
    assert rho > 0.9, rho
    # the measured prefix frequency estimates the generator's mean there
    assert cal.hot_p_mean == pytest.approx(float(p_new[:192].mean()), rel=0.1)


def test_calibration_of_a_sorted_layer_keeps_its_head():
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=256, f=640, r=64)
    lt = inputs.make_layer(cfg, 0, seed=2)
    L = _host(lt)
    batches = [_u(cfg, step, 64, 2) for step in range(8)]
    lr, cal = calibrate.calibrate_layer(lt, lambda u: oracle.predict(L, u.numpy())["idx"], batches, frac=0.2)
    # the generator's hot prefix and the measured one are mostly the same neurons
    H = lt.hot_prefix
    assert cal.hot_prefix == (H // 32) * 32
    assert len(set(cal.perm[:H].tolist()) & set(range(H))) >= 0.85 * H


def test_hot_prefix_rules():
    f = 256
    assert calibrate.hot_prefix_for_batch(np.ones(f), 1) == f
    assert calibrate.hot_prefix_for_batch(np.zeros(f), 8) == 0
    half = np.full(f, 0.5)
    assert calibrate.hot_prefix_for_batch(half, 1) == 0      # 0.5 < 0.75
    assert calibrate.hot_prefix_for_batch(half, 2) == f      # 1 - 0.25 = 0.75
    q = np.concatenate([np.full(100, 0.9), np.full(156, 0.1)])
    assert calibrate.hot_prefix_for_batch(q, 1) == 96        # 100 rounded down to 32
    assert calibrate.hot_prefix_for_batch(q, 1, union=0.95) == 0
    assert calibrate.hot_prefix_for_batch(q, 32) == f        # 1 - 0.9^32 = 0.966
    with pytest.raises(ValueError):
        calibrate.hot_prefix_for_batch(q[::-1], 1)
    assert calibrate.hot_prefix_fraction(16384, 0.2) == 3264
    assert calibrate.hot_prefix_fraction(1000, 0.2) == 192


def test_firing_counts_validates_predictor_output():
    u = torch.zeros(2, 8)
    with pytest.raises(ValueError):
        calibrate.firing_counts(lambda u: [np.array([1])], [u], 16)
    with pytest.raises(ValueError):
        calibrate.firing_counts(lambda u: [np.array([1, 1]), np.array([])], [u], 16)
    with pytest.raises(ValueError):
        calibrate.firing_counts(lambda u: [np.array([16]), np.array([])], [u], 16)
    c, n = calibrate.firing_counts(lambda u: [np.array([0, 3]), np.array([3])], [u, u], 4)
    assert n == 4 and c.tolist() == [2, 0, 0, 4]


# ---------------------------------------------------------------- predictor sizing

def test_truncate_predictor_keeps_leading_components():
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=128, f=256, r=64)
    lt = inputs.make_layer(cfg, 0, seed=5)
    t = calibrate.truncate_predictor(lt, 16)
    assert t.r == 16 and t.p1.shape == (16, 128) and t.p2.shape == (256, 16)
    assert torch.equal(t.p1, lt.p1[:16]) and torch.equal(t.p2, lt.p2[:, :16])
    assert torch.equal(t.p_bias, lt.p_bias) and torch.equal(t.w_up, lt.w_up)
    assert torch.equal(calibrate.truncate_predictor(lt, 64).p2, lt.p2)
    for bad in (0, 65):
        with pytest.raises(ValueError):
            calibrate.truncate_predictor(lt, bad)
    # the factors are in descending singular-value order: the leading
    # component of P2 carries the most energy
    col = torch.linalg.vector_norm(lt.p2.double(), dim=0)
    assert torch.all(col[:-1] >= col[1:] - 1e-3)


def test_cosine_shift_and_recall_closed_forms():
    y = np.array([[1.0, 0.0], [0.0, 0.0], [1.0, 1.0], [0.0, 0.0]])
    r = np.array([[2.0, 0.0], [0.0, 0.0], [1.0, -1.0], [1.0, 0.0]])
    assert np.allclose(calibrate.cosine_shift(y, r), [0.0, 0.0, 1.0, 1.0])
    assert calibrate.set_recall([np.array([1, 2, 3])], [np.array([2, 3, 4, 5])]) == 0.5
    assert calibrate.set_recall([np.array([], np.int32)], [np.array([], np.int32)]) == 1.0


def test_size_rank_against_the_exact_relu_mask():
    """On a small ReLU layer, the sizing compares each truncated predictor's
    outputs with those over the exact mask (pre-activation > 0): the shift
    falls as the rank grows, the full-rank predictor is within the pages'
    0.4% shift, and the choice is the smallest rank that meets the target."""
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=128, f=512, r=128)
    lt = inputs.make_layer(cfg, 0, seed=9)
    L = _host(lt)
    hosts = {r: _host(calibrate.truncate_predictor(lt, r)) for r in (8, 32, 128)}
    batches = [_u(cfg, step, 32, 9) for step in range(2)]

    def predict_at(r, u):
        return oracle.predict(hosts[r], u.numpy())["idx"]

    def ffn(u, sets):
        return oracle.ffn_masked(L, u.numpy(), sets)

    def exact(u):
        pre = oracle.relu_preact(L, u.numpy())
        return [np.nonzero(p > 0)[0].astype(np.int32) for p in pre]

    ch = calibrate.size_rank([8, 32, 128], predict_at, ffn, exact, batches)
    shifts = [row["mean_shift"] for row in ch.table]
    assert shifts[0] > shifts[1] > shifts[2]
    assert ch.table[2]["mean_shift"] <= 0.004 and ch.table[2]["recall"] > 0.95
    assert ch.met and ch.rank == min(row["rank"] for row in ch.table if row["mean_shift"] <= 0.004)
    loose = calibrate.size_rank([8, 32, 128], predict_at, ffn, exact, batches, max_shift=1.0)
    assert loose.rank == 8 and loose.met
    none = calibrate.size_rank([8, 32], predict_at, ffn, exact, batches, max_shift=-1.0)
    assert none.rank == 32 and not none.met
