"""Seeded synthetic workloads: FFN layer weights, predictor factors and tokens.

This module only *makes inputs*.  It evaluates no step of the decode path
(no predictor score, no FFN, no normalisation); the CUDA library and the CPU
oracle both consume what it returns.

Workload recipe (the pages evaluate trained OPT / LLaMA2 models on public
datasets; none are available, so seeded synthetic layers with the same FFN
shapes stand in for them):

* weights ~ N(0, 0.02^2), each (config, layer, tensor) independently seeded;
* firing probability of the neuron with popularity rank k (0 = hottest):
  p = min(c * (k+1)^-0.8, 0.99); c is either given (0.5 for the small fp32
  layer) or found by bisection so that mean(p) hits the config's target
  sparsity (the power-law activation locality of the pages' Summary; the
  measured sparsities of the Key points: 97% OPT-30B, 43% LLaMA2-13B);
* predictor = rank-r truncated SVD of the up (ReLU) or gate (SwiGLU) weights
  as the layer stores them: P1 = V_r^T [r x d], P2 = U_r Sigma_r [f x r]
  (exact SVD for small layers, a seeded randomized range finder with two
  power iterations for large ones; the stored factors define the predictor,
  so SVD accuracy does not matter);
* predictor bias b_i = sigma_i * Phi^-1(p_i) with sigma_i = ||(P2 P1)_i|| (the
  predictor row norm) so that, for u ~ N(0, I), neuron i is predicted active
  with probability p_i.  ``bias_norm="w1"`` uses ||W1_i|| instead.  For ReLU
  layers the same vector is the FFN bias b1;
* neurons are reordered by descending p (the offline hot/cold reordering of
  the pages' Interesting ideas I1), so the hot prefix [0, H), H = 0.2 f, is a
  contiguous block; the small fp32 layer keeps its seeded random order;
* int4 weights: per 32-element group along d, scale = fp16(absmax / 7),
  q = clamp(rne(w / scale), -8, 7) + 8, element 2k in the low nibble of byte k;
* tokens: x ~ N(0, I) per decode step; single-layer fp16 configs feed
  u = fp16(x) directly, the fp32 layer feeds u = x.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np
import torch


# --------------------------------------------------------------------------
# configurations (the five workload shapes)
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Config:
    name: str
    d: int                  # d_model
    f: int                  # d_ffn (neurons)
    r: int                  # predictor rank
    n_layers: int
    act: str                # "relu" | "swiglu"
    wtype: str              # "f32" | "f16" | "int4g32"
    mean_p: Optional[float]  # target mean firing probability (None: use c)
    c: Optional[float] = None
    sort_neurons: bool = True
    hot_frac: float = 0.2
    batches: Tuple[int, ...] = (1,)
    tokens: int = 64
    stacked: bool = False
    w_std: float = 0.02
    bias_norm: str = "pred"  # "pred" | "w1"

    def scaled(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, Config] = {
    # single OPT-style ReLU layer, fp32, literal power law c = 0.5, random order
    "opt_tiny_f32": Config("opt_tiny_f32", d=256, f=1024, r=32, n_layers=1, act="relu", wtype="f32",
                           mean_p=None, c=0.5, sort_neurons=False, batches=(1,), tokens=64),
    # OPT-7B-shaped ReLU layer, fp16, mean p 10%, hot prefix 20%
    "opt7b_f16": Config("opt7b_f16", d=4096, f=16384, r=1024, n_layers=1, act="relu", wtype="f16",
                        mean_p=0.10, batches=(1, 8), tokens=256),
    # OPT-30B-shaped 48-layer ReLU stack, fp16, mean p 3%
    "opt30b_stack_f16": Config("opt30b_stack_f16", d=7168, f=28672, r=1024, n_layers=48, act="relu",
                               wtype="f16", mean_p=0.03, batches=(1,), tokens=128, stacked=True),
    # LLaMA2-13B-shaped 40-layer SwiGLU stack, fp16, 43% predicted active
    "llama13b_swiglu_f16": Config("llama13b_swiglu_f16", d=5120, f=13824, r=1024, n_layers=40, act="swiglu",
                                  wtype="f16", mean_p=0.43, batches=(1, 4), tokens=64, stacked=True),
    # LLaMA2-70B-shaped 80-layer SwiGLU stack, int4 groups of 32, 50% predicted active
    "llama70b_swiglu_int4": Config("llama70b_swiglu_int4", d=8192, f=28672, r=1024, n_layers=80,
                                   act="swiglu", wtype="int4g32", mean_p=0.50, batches=(1, 4, 16, 32),
                                   tokens=32, stacked=True),
}
CONFIG_ORDER = list(CONFIGS)


# --------------------------------------------------------------------------
# seeds
# --------------------------------------------------------------------------

def derive_seed(*parts) -> int:
    """Stable 63-bit seed from any printable parts (independent of PYTHONHASHSEED)."""
    h = hashlib.sha256("|".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(*parts))
    return g


# --------------------------------------------------------------------------
# firing probabilities
# --------------------------------------------------------------------------

def power_law(f: int, c: float, exponent: float = 0.8, cap: float = 0.99) -> np.ndarray:
    k = np.arange(1, f + 1, dtype=np.float64)
    return np.minimum(c * k ** (-exponent), cap)


def calibrate_c(f: int, mean_p: float, exponent: float = 0.8, cap: float = 0.99) -> float:
    lo, hi = 0.0, 1.0
    while power_law(f, hi, exponent, cap).mean() < mean_p:
        hi *= 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if power_law(f, mid, exponent, cap).mean() < mean_p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def firing_probs(cfg: Config) -> np.ndarray:
    """p by popularity rank (index 0 = hottest)."""
    c = cfg.c if cfg.mean_p is None else calibrate_c(cfg.f, cfg.mean_p)
    return power_law(cfg.f, c)


# --------------------------------------------------------------------------
# int4 group quantiser
# --------------------------------------------------------------------------

def quantize_int4g32(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """w [rows x d] float -> (packed uint8 [rows x d/2], fp16 scales [rows x d/32],
    dequantised float32 [rows x d])."""
    rows, d = w.shape
    assert d % 32 == 0
    g = w.float().reshape(rows, d // 32, 32)
    scale = (g.abs().amax(dim=2) / 7.0).to(torch.float16)
    sf = scale.float().unsqueeze(2)
    safe = torch.where(sf == 0, torch.ones_like(sf), sf)
    q = torch.clamp(torch.round(g / safe), -8, 7)        # torch.round: half to even
    q = torch.where(sf == 0, torch.zeros_like(q), q) + 8
    q = q.to(torch.uint8).reshape(rows, d)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).contiguous()
    deq = (sf * (q.reshape(rows, d // 32, 32).float() - 8.0)).reshape(rows, d)
    return packed, scale.contiguous(), deq


# --------------------------------------------------------------------------
# predictor factors
# --------------------------------------------------------------------------

def _svd_factors(w: torch.Tensor, r: int, gen_device, seed_parts) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rank-r truncated SVD of w [f x d]: (P1 = V_r^T [r x d], P2 = U_r S_r [f x r]) in fp64/fp32."""
    f, d = w.shape
    if f * d <= (1 << 22) or r >= min(f, d):
        W = w.double()
        U, S, Vh = torch.linalg.svd(W, full_matrices=False)
        return Vh[:r].contiguous(), (U[:, :r] * S[:r]).contiguous()
    # randomized range finder (Halko, Martinsson & Tropp 2011) with a seeded sketch
    W = w.float()
    g = _gen(gen_device, *seed_parts, "sketch")
    omega = torch.randn(d, r, generator=g, device=W.device, dtype=torch.float32)
    Q, _ = torch.linalg.qr(W @ omega)
    for _ in range(2):
        Z, _ = torch.linalg.qr(W.T @ Q)
        Q, _ = torch.linalg.qr(W @ Z)
    Bm = (Q.T @ W).double()                                   # [r x d]
    evals, Uh = torch.linalg.eigh(Bm @ Bm.T)                  # ascending
    order = torch.argsort(evals, descending=True)
    evals, Uh = evals[order].clamp_min(0), Uh[:, order]
    S = evals.sqrt()
    Vh = (Uh.T @ Bm) / S.clamp_min(1e-30).unsqueeze(1)        # [r x d], rows orthonormal
    P2 = (Q.double() @ Uh) * S                                # [f x r]
    return Vh.contiguous(), P2.contiguous()


# --------------------------------------------------------------------------
# one layer
# --------------------------------------------------------------------------

@dataclass
class LayerTensors:
    """One FFN layer and its predictor, as stored on ``device``.

    Per-neuron arrays are in storage order (hot prefix first when sorted).
    """
    cfg: Config
    layer: int
    w_up: torch.Tensor                 # ReLU: W1; SwiGLU: W_up.  [f x d] (int4: uint8 [f x d/2])
    w_down_t: torch.Tensor             # W2^T, neuron-major
    p1: torch.Tensor                   # [r x d]
    p2: torch.Tensor                   # [f x r]
    p_bias: torch.Tensor               # [f] fp32
    b_up: Optional[torch.Tensor] = None    # ReLU bias b1 [f] fp32 (same values as p_bias)
    w_gate: Optional[torch.Tensor] = None
    s_up: Optional[torch.Tensor] = None    # int4 scales fp16 [f x d/32]
    s_gate: Optional[torch.Tensor] = None
    s_down_t: Optional[torch.Tensor] = None
    p: Optional[np.ndarray] = None         # firing probability per stored neuron
    hot_prefix: int = 0
    hot_p_mean: float = 0.0
    extra: Dict[str, object] = field(default_factory=dict)

    @property
    def d(self):
        return self.cfg.d

    @property
    def f(self):
        return self.cfg.f

    @property
    def r(self):
        return self.cfg.r

    def tensors(self) -> Dict[str, Optional[torch.Tensor]]:
        return dict(w_up=self.w_up, w_gate=self.w_gate, w_down_t=self.w_down_t, s_up=self.s_up,
                    s_gate=self.s_gate, s_down_t=self.s_down_t, b_up=self.b_up, p1=self.p1, p2=self.p2,
                    p_bias=self.p_bias)

    def to(self, device) -> "LayerTensors":
        kw = {k: (None if v is None else v.to(device)) for k, v in self.tensors().items()}
        return dataclasses.replace(self, **kw)

    def host_arrays(self) -> Dict[str, object]:
        """numpy copies with the oracle's field names (fp16 stays float16)."""
        out = dict(d=self.d, f=self.f, r=self.r, act=self.cfg.act, wtype=self.cfg.wtype)
        for k, v in self.tensors().items():
            out[k] = None if v is None else v.detach().cpu().numpy()
        return out

    def nbytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.tensors().values() if v is not None)


def _wdtype(cfg: Config):
    return torch.float32 if cfg.wtype == "f32" else torch.float16


def make_layer(cfg: Config, layer: int = 0, seed: int = 0, device="cpu") -> LayerTensors:
    dev = torch.device(device)
    gdev = dev.type if dev.type == "cpu" else dev
    tag = (seed, cfg.name, cfg.d, cfg.f, cfg.r, layer)
    d, f, r = cfg.d, cfg.f, cfg.r

    def randn(name, shape):
        g = _gen(gdev, *tag, name)
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32) * cfg.w_std

    names = ["w_up", "w_down_t"] + (["w_gate"] if cfg.act == "swiglu" else [])
    stored, scales, deq = {}, {}, {}
    for n in names:
        w = randn(n, (f, d))
        if cfg.wtype == "int4g32":
            stored[n], scales[n], deq[n] = quantize_int4g32(w)
        else:
            stored[n] = w.to(_wdtype(cfg)).contiguous()
            deq[n] = stored[n].float()
        del w
    src = deq["w_up"] if cfg.act == "relu" else deq["w_gate"]
    p1, p2 = _svd_factors(src, r, gdev, tag)
    ptype = torch.float32 if cfg.wtype == "f32" else torch.float16
    p1s, p2s = p1.to(ptype).contiguous(), p2.to(ptype).contiguous()

    # firing probabilities under a seeded popularity ranking, and the bias
    p_by_rank = firing_probs(cfg)
    g = _gen("cpu", *tag, "rank")
    rank = torch.randperm(f, generator=g).numpy()          # rank of neuron i
    p = p_by_rank[rank]
    if cfg.bias_norm == "pred":
        P1d = p1s.double()
        G = P1d @ P1d.T
        P2d = p2s.double()
        sigma = torch.sqrt(((P2d @ G) * P2d).sum(dim=1)).cpu().numpy()
    else:
        sigma = torch.linalg.vector_norm(src.double(), dim=1).cpu().numpy()
    z = torch.special.ndtri(torch.from_numpy(p).double()).numpy()
    bias = torch.from_numpy((sigma * z).astype(np.float32)).to(dev)
    del src, deq

    # offline reordering: storage order = descending p (= ascending rank)
    if cfg.sort_neurons:
        perm_np = np.argsort(rank, kind="stable")
        perm = torch.from_numpy(perm_np).to(dev)
        for n in names:
            stored[n] = stored[n].index_select(0, perm).contiguous()
            if n in scales:
                scales[n] = scales[n].index_select(0, perm).contiguous()
        p2s = p2s.index_select(0, perm).contiguous()
        bias = bias.index_select(0, perm).contiguous()
        p = p[perm_np]
        H = int(math.floor(cfg.hot_frac * f))
    else:
        H = 0
    lt = LayerTensors(cfg=cfg, layer=layer, w_up=stored["w_up"], w_down_t=stored["w_down_t"], p1=p1s, p2=p2s,
                      p_bias=bias, b_up=bias if cfg.act == "relu" else None, w_gate=stored.get("w_gate"),
                      s_up=scales.get("w_up"), s_gate=scales.get("w_gate"), s_down_t=scales.get("w_down_t"),
                      p=p, hot_prefix=H, hot_p_mean=float(p[:H].mean()) if H else 0.0)
    return lt


def make_tokens(cfg: Config, step: int, B: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """x ~ N(0, I) [B x d] fp32 for decode step ``step``."""
    dev = torch.device(device)
    g = _gen(dev.type if dev.type == "cpu" else dev, seed, cfg.name, cfg.d, "x", step, B)
    return torch.randn((B, cfg.d), generator=g, device=dev, dtype=torch.float32)


def layer_input(cfg: Config, x: torch.Tensor) -> torch.Tensor:
    """FFN input u of a single (unstacked) layer: x itself (fp32 layer) or fp16(x)."""
    return x.contiguous() if cfg.wtype == "f32" else x.to(torch.float16).contiguous()


# --------------------------------------------------------------------------
# exact-arithmetic layers (every sum exact in fp32: small integers x 2^-k)
# --------------------------------------------------------------------------

def make_exact_layer(d: int, f: int, r: int, act: str = "relu", wtype: str = "f16", seed: int = 0,
                     device="cpu", hot_frac: float = 0.2) -> LayerTensors:
    """Weights in {-3..3} * 2^-4, predictor factors in {-2..2} * 2^-3, bias in
    {-8..8} * 2^-4, int4 scales powers of two.  With small-integer u, every
    product and partial sum is a multiple of 2^-11 of modest size, so fp32 and
    double sums agree exactly in any order (including exact zeros)."""
    dev = torch.device(device)
    gdev = dev.type if dev.type == "cpu" else dev
    tag = ("exact", seed, d, f, r, act, wtype)

    def ints(name, shape, lo, hi):
        g = _gen(gdev, *tag, name)
        return torch.randint(lo, hi + 1, shape, generator=g, device=dev).float()

    cfg = Config("exact", d=d, f=f, r=r, n_layers=1, act=act, wtype=wtype, mean_p=None, c=0.5,
                 sort_neurons=True, hot_frac=hot_frac)
    names = ["w_up", "w_down_t"] + (["w_gate"] if act == "swiglu" else [])
    stored, scales = {}, {}
    for n in names:
        if wtype == "int4g32":
            q = ints(n, (f, d), 0, 15).to(torch.uint8)
            e = ints(n + "_e", (f, d // 32), -6, -3)
            scales[n] = torch.pow(2.0, e).to(torch.float16).contiguous()
            stored[n] = (q[:, 0::2] | (q[:, 1::2] << 4)).contiguous()
        else:
            stored[n] = (ints(n, (f, d), -3, 3) / 16.0).to(_wdtype(cfg)).contiguous()
    pt = torch.float32 if wtype == "f32" else torch.float16
    p1 = (ints("p1", (r, d), -2, 2) / 8.0).to(pt).contiguous()
    p2 = (ints("p2", (f, r), -2, 2) / 8.0).to(pt).contiguous()
    bias = (ints("bias", (f,), -8, 8) / 16.0).contiguous()
    H = int(math.floor(hot_frac * f))
    return LayerTensors(cfg=cfg, layer=0, w_up=stored["w_up"], w_down_t=stored["w_down_t"], p1=p1, p2=p2,
                        p_bias=bias, b_up=bias if act == "relu" else None, w_gate=stored.get("w_gate"),
                        s_up=scales.get("w_up"), s_gate=scales.get("w_gate"), s_down_t=scales.get("w_down_t"),
                        p=np.full(f, 0.5), hot_prefix=H, hot_p_mean=0.5)


def make_exact_tokens(d: int, B: int, step: int = 0, seed: int = 0, device="cpu", dtype=torch.float16):
    """u with small-integer entries in {-4..4} (exact in fp16)."""
    dev = torch.device(device)
    g = _gen(dev.type if dev.type == "cpu" else dev, "exact-u", seed, d, B, step)
    return torch.randint(-4, 5, (B, d), generator=g, device=dev).to(dtype).contiguous()
