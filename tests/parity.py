"""Shared parity checks: CUDA path (through the C ABI) against the CPU oracle.

Contract (what the decode path must reproduce):
  * active sets: for every neuron whose oracle score lies outside the
    oracle's rounding band (|s_i| > band_i) the GPU decision is identical;
    inside the band either decision is correct.  The band must stay below 1%
    of the neurons.
  * outputs: max |y_gpu - y_ref| / max |y_ref| <= 1e-5 for fp32 layers and
    <= 2e-3 for fp16 / int4 layers (fp32 accumulation); when y_ref is
    identically zero, y_gpu must be exactly zero.
  * y_ref is the oracle's masked sum over the set being checked: the
    oracle's own set, or, for the fused decode step, the oracle's set with
    the in-band neurons decided as the GPU decided them (each such neuron is
    individually valid per the band rule; the oracle evaluates its term).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import inputs

TOL = {"f32": 1e-5, "f16": 2e-3, "int4g32": 2e-3}


def host_layer(lt: inputs.LayerTensors) -> oracle.Layer:
    return oracle.Layer(**lt.host_arrays())


def rel_err(y_gpu: np.ndarray, y_ref: np.ndarray) -> float:
    den = np.max(np.abs(y_ref))
    num = np.max(np.abs(y_gpu.astype(np.float64) - y_ref))
    if den == 0:
        return 0.0 if num == 0 else np.inf
    return num / den


def assert_outputs(y_gpu: np.ndarray, y_ref: np.ndarray, wtype: str, what=""):
    for b in range(y_ref.shape[0]):
        den = np.max(np.abs(y_ref[b]))
        if den == 0:
            assert np.all(y_gpu[b] == 0), f"{what} token {b}: reference is zero, GPU is not"
        else:
            e = rel_err(y_gpu[b], y_ref[b])
            assert e <= TOL[wtype], f"{what} token {b}: rel err {e:.3e} > {TOL[wtype]}"


def gpu_sets(idx: torch.Tensor, count: torch.Tensor):
    idx, count = idx.cpu().numpy(), count.cpu().numpy()
    return [idx[b, :count[b]].copy() for b in range(len(count))]


def compare_sets(gpu, pr, f):
    """Check GPU sets against the oracle's prediction outside the band.
    Returns (sets to evaluate y on, number of in-band flips, band fraction)."""
    out, flips, band_pop = [], 0, 0
    for b, g in enumerate(gpu):
        assert np.all(np.diff(g) > 0), "GPU id list not strictly ascending"
        assert len(g) == 0 or (g[0] >= 0 and g[-1] < f)
        s, band = pr["s"][b], pr["band"][b]
        amb = np.abs(s) <= band
        gm = np.zeros(f, bool)
        gm[g] = True
        om = s > 0
        bad = (gm != om) & ~amb
        assert not np.any(bad), f"token {b}: {int(bad.sum())} out-of-band mismatches, e.g. ids {np.nonzero(bad)[0][:8]}"
        flips += int(np.sum((gm != om) & amb))
        band_pop += int(amb.sum())
        if np.any(gm != om):
            m = om.copy()          # oracle's set, in-band neurons decided as the GPU did
            m[amb] = gm[amb]
            out.append(np.nonzero(m)[0].astype(np.int32))
        else:
            out.append(pr["idx"][b])
    frac = band_pop / (f * len(gpu))
    assert frac < 0.01, f"rounding band covers {frac:.4f} of neurons"
    return out, flips, frac


class Gpu:
    """A layer on the device with its handle and a workspace."""

    def __init__(self, lt: inputs.LayerTensors, max_batch: int, device="cuda"):
        self.lt = lt.to(device)
        self.layer = pb.FfnLayer.from_tensors(self.lt)
        self.ws = pb.make_workspace([self.layer], max_batch, device)

    def predict(self, u: torch.Tensor):
        B = u.shape[0]
        idx = torch.full((B, self.lt.f), -7, dtype=torch.int32, device=u.device)
        cnt = torch.full((B,), -7, dtype=torch.int32, device=u.device)
        pb.pi_predict(self.layer, u, idx, cnt, self.ws)
        return idx, cnt

    def sparse_ffn(self, u: torch.Tensor, sets, flags=0):
        B = u.shape[0]
        idx = torch.zeros((B, self.lt.f), dtype=torch.int32)
        cnt = torch.zeros(B, dtype=torch.int32)
        for b, s in enumerate(sets):
            idx[b, :len(s)] = torch.from_numpy(np.asarray(s, np.int32))
            cnt[b] = len(s)
        y = torch.full((B, self.lt.d), float("nan"), device=u.device)
        pb.pi_sparse_ffn(self.layer, u, idx.to(u.device), cnt.to(u.device), y, self.ws, flags=flags)
        return y

    def decode(self, u: torch.Tensor, flags=0):
        B = u.shape[0]
        idx = torch.full((B, self.lt.f), -7, dtype=torch.int32, device=u.device)
        cnt = torch.full((B,), -7, dtype=torch.int32, device=u.device)
        y = torch.full((B, self.lt.d), float("nan"), device=u.device)
        pb.pi_decode_ffn(self.layer, u, y, self.ws, idx=idx, count=cnt, flags=flags)
        return y, idx, cnt

    def status(self) -> int:
        return pb.pi_get_device_status(self.ws)


def check_layer(lt: inputs.LayerTensors, u_host: torch.Tensor, gpu: Gpu, flags=0):
    """Full parity of one layer on one batch: predict, sparse FFN on the
    oracle's sets, fused decode.  Returns a small report dict."""
    L = host_layer(lt)
    u_np = u_host.numpy()
    pr = oracle.predict(L, u_np)
    u_dev = u_host.to("cuda")
    # predictor
    idx, cnt = gpu.predict(u_dev)
    sets, flips, frac = compare_sets(gpu_sets(idx, cnt), pr, lt.f)
    # sparse FFN on the oracle's own sets
    y_ref = oracle.ffn_masked(L, u_np, pr["idx"])
    y = gpu.sparse_ffn(u_dev, pr["idx"], flags=flags).cpu().numpy()
    assert_outputs(y, y_ref, lt.cfg.wtype, "pi_sparse_ffn")
    # fused decode step
    yd, idx2, cnt2 = gpu.decode(u_dev, flags=flags)
    sets2, flips2, _ = compare_sets(gpu_sets(idx2, cnt2), pr, lt.f)
    y_ref2 = y_ref if flips2 == 0 else oracle.ffn_masked(L, u_np, sets2)
    assert_outputs(yd.cpu().numpy(), y_ref2, lt.cfg.wtype, "pi_decode_ffn")
    assert gpu.status() == 0
    return dict(flips=flips + flips2, band_frac=frac, count=pr["count"].tolist(),
                err=max(rel_err(y[b], y_ref[b]) for b in range(len(y))))
