"""Offline hot/cold reordering from measured firing frequencies.

PowerInfer summary page, Summary (second paragraph) and Interesting ideas I1:
an offline pass runs the model on calibration inputs, records how often each
neuron is used, and lays the frequently used neurons out where they are
cheapest to read.  Here the record is the predictor's firing count per
neuron over calibration tokens, and the layout is the storage order: the
most frequently predicted neurons first, so that the hot prefix [0, H) is one
contiguous block that the kernels may read densely (the dense/index choice
of ``pi_ffn_desc.hot_prefix`` and ``hot_p_mean``).

Nothing here computes a step of the decode path.  ``firing_counts`` takes
the predictor as a callable, e.g. the library's own ``pi_predict``::

    layer = binding.FfnLayer.from_tensors(lt_on_device)
    ws = binding.make_workspace([layer], max_batch)
    def predict(u):                       # u: [B x d] on the device
        idx = torch.empty((u.shape[0], lt.f), dtype=torch.int32, device=u.device)
        cnt = torch.empty(u.shape[0], dtype=torch.int32, device=u.device)
        binding.pi_predict(layer, u, idx, cnt, ws)
        idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
        return [idx[b, :cnt[b]] for b in range(len(cnt))]

Reordering permutes the neuron axis of every per-neuron tensor (up, gate and
down rows, their int4 scales, the P2 rows and the biases) by one
permutation; P1 is not per neuron and stays.  The FFN output is a sum over
neurons, so it is unchanged up to the order of that sum, and a token's
predicted set maps through the permutation.

Predictor sizing (the summary page's Interesting ideas I3: each layer's
predictor is sized by how predictable the layer is, within an accuracy
target; its Key points quote a ~0.4% cosine shift of the layer outputs for
the trained predictors): ``truncate_predictor`` keeps the leading r
components of the factors, and ``size_rank`` picks the smallest candidate
rank whose outputs stay within a mean cosine shift of a reference (the
exact ReLU mask, or the full predictor) on calibration tokens.  The FFN
evaluator and the predictors are callables again: the library's
pi_predict / pi_sparse_ffn on the device, or the oracle in the tests.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Iterable, List, Sequence

import numpy as np
import torch

from .inputs import LayerTensors

ALIGN = 32  # the hot prefix is a whole number of 32-neuron mask words
DENSE_UNION = 0.75  # union density at which the library reads the prefix densely


def firing_counts(predict: Callable[[torch.Tensor], Sequence[np.ndarray]], batches: Iterable[torch.Tensor],
                  f: int) -> tuple[np.ndarray, int]:
    """Per-neuron firing counts over calibration batches.

    ``predict(u)`` returns one array of fired neuron ids per token of ``u``.
    Returns (counts [f] int64, number of tokens seen)."""
    counts = np.zeros(f, np.int64)
    n = 0
    for u in batches:
        sets = predict(u)
        if len(sets) != u.shape[0]:
            raise ValueError(f"predict returned {len(sets)} sets for {u.shape[0]} tokens")
        for s in sets:
            s = np.asarray(s, np.int64)
            if s.size and (s.min() < 0 or s.max() >= f or np.unique(s).size != s.size):
                raise ValueError("predicted ids must be distinct and in [0, f)")
            counts[s] += 1
        n += len(sets)
    return counts, n


def hot_order(counts: np.ndarray) -> np.ndarray:
    """Storage order: neurons by descending count, ties kept in their current
    order (stable).  ``perm[k]`` is the current index of the neuron stored at k."""
    return np.argsort(-np.asarray(counts, np.int64), kind="stable")


def hot_prefix_for_batch(freq_sorted: np.ndarray, batch: int, union: float = DENSE_UNION,
                         align: int = ALIGN) -> int:
    """Largest H (a multiple of ``align``) such that every neuron in [0, H)
    is expected in the union of ``batch`` tokens with probability >= ``union``
    (1 - (1 - q)^batch >= union for its measured frequency q): reading those
    rows densely wastes at most 1 - union of them.  ``freq_sorted`` must be
    non-increasing."""
    q = np.asarray(freq_sorted, np.float64)
    if q.size and np.any(np.diff(q) > 0):
        raise ValueError("frequencies must be sorted in non-increasing order")
    if batch < 1 or not (0.0 < union <= 1.0):
        raise ValueError("batch >= 1 and 0 < union <= 1 required")
    ok = 1.0 - np.power(1.0 - np.clip(q, 0.0, 1.0), batch) >= union
    n = int(np.argmin(ok)) if not ok.all() else q.size  # ok is a prefix of True values
    return (n // align) * align


def hot_prefix_fraction(f: int, frac: float, align: int = ALIGN) -> int:
    """H = floor(frac * f), rounded down to a multiple of ``align``."""
    if not (0.0 <= frac <= 1.0):
        raise ValueError("0 <= frac <= 1 required")
    return (int(np.floor(frac * f)) // align) * align


def reorder_layer(lt: LayerTensors, perm: np.ndarray, hot_prefix: int = 0,
                  hot_p_mean: float = 0.0) -> LayerTensors:
    """The layer with its neurons stored in the order ``perm`` (new k = old
    perm[k]), and the given hot-prefix description."""
    perm = np.asarray(perm, np.int64)
    if perm.shape != (lt.f,) or not np.array_equal(np.sort(perm), np.arange(lt.f)):
        raise ValueError("perm must be a permutation of range(f)")
    if hot_prefix < 0 or hot_prefix > lt.f or hot_prefix % ALIGN:
        raise ValueError(f"hot_prefix must be a multiple of {ALIGN} in [0, f]")
    kw = {}
    for name in ("w_up", "w_gate", "w_down_t", "s_up", "s_gate", "s_down_t", "p2", "p_bias"):
        t = getattr(lt, name)
        kw[name] = None if t is None else t.index_select(0, torch.from_numpy(perm).to(t.device)).contiguous()
    # the ReLU bias b1 is the same vector as the predictor bias
    kw["b_up"] = kw["p_bias"] if lt.b_up is not None else None
    kw["p"] = None if lt.p is None else lt.p[perm]
    return dataclasses.replace(lt, hot_prefix=int(hot_prefix), hot_p_mean=float(hot_p_mean), **kw)


@dataclasses.dataclass
class Calibration:
    perm: np.ndarray         # new storage order (indices into the input layer)
    counts: np.ndarray       # firing counts in the new order (non-increasing)
    tokens: int              # calibration tokens seen
    hot_prefix: int
    hot_p_mean: float        # mean measured frequency of [0, hot_prefix)


def calibrate_layer(lt: LayerTensors, predict: Callable[[torch.Tensor], Sequence[np.ndarray]],
                    batches: Iterable[torch.Tensor], batch: int = 1, union: float = DENSE_UNION,
                    frac: float | None = None) -> tuple[LayerTensors, Calibration]:
    """Measure firing frequencies with ``predict`` on ``batches``, store the
    neurons hot-first, and size the hot prefix: by ``frac`` of f when given,
    else as the prefix that ``batch`` tokens cover densely
    (``hot_prefix_for_batch``)."""
    counts, n = firing_counts(predict, batches, lt.f)
    if n == 0:
        raise ValueError("no calibration tokens")
    perm = hot_order(counts)
    c = counts[perm]
    q = c / float(n)
    H = hot_prefix_fraction(lt.f, frac) if frac is not None else hot_prefix_for_batch(q, batch, union)
    pm = float(q[:H].mean()) if H else 0.0
    return reorder_layer(lt, perm, H, pm), Calibration(perm=perm, counts=c, tokens=n, hot_prefix=H, hot_p_mean=pm)


def map_sets(sets: List[np.ndarray], perm: np.ndarray) -> List[np.ndarray]:
    """Predicted sets of the original layer expressed in the reordered
    layer's ids (ascending)."""
    inv = np.empty_like(np.asarray(perm, np.int64))
    inv[perm] = np.arange(len(perm))
    return [np.sort(inv[np.asarray(s, np.int64)]).astype(np.int32) for s in sets]


# --------------------------------------------------------------------------
# predictor sizing
# --------------------------------------------------------------------------

def truncate_predictor(lt: LayerTensors, rank: int) -> LayerTensors:
    """The layer with a rank-``rank`` predictor: the leading ``rank`` rows of
    P1 and columns of P2.  The generator's factors are P1 = V_r^T and
    P2 = U_r Sigma_r of a truncated SVD in descending singular-value order, so
    the cut is the rank-``rank`` truncated SVD of the same matrix.  The bias
    and every FFN tensor stay."""
    if rank < 1 or rank > lt.r:
        raise ValueError(f"rank must be in [1, {lt.r}]")
    cfg = dataclasses.replace(lt.cfg, r=int(rank))
    return dataclasses.replace(lt, cfg=cfg, p1=lt.p1[:rank].contiguous(), p2=lt.p2[:, :rank].contiguous())


def cosine_shift(y: np.ndarray, y_ref: np.ndarray) -> np.ndarray:
    """1 - cos(y_b, y_ref_b) per token (0 where both are zero, 1 where only one is)."""
    y, y_ref = np.atleast_2d(np.asarray(y, np.float64)), np.atleast_2d(np.asarray(y_ref, np.float64))
    num = np.sum(y * y_ref, axis=1)
    den = np.linalg.norm(y, axis=1) * np.linalg.norm(y_ref, axis=1)
    both0 = (np.linalg.norm(y, axis=1) == 0) & (np.linalg.norm(y_ref, axis=1) == 0)
    out = np.where(den > 0, 1.0 - num / np.where(den > 0, den, 1.0), 1.0)
    return np.where(both0, 0.0, out)


def set_recall(pred: Sequence[np.ndarray], ref: Sequence[np.ndarray]) -> float:
    """Mean over tokens of |pred & ref| / |ref| (tokens with an empty ref count as 1)."""
    vals = []
    for p, r in zip(pred, ref):
        r = np.asarray(r)
        vals.append(1.0 if r.size == 0 else np.intersect1d(np.asarray(p), r).size / r.size)
    return float(np.mean(vals)) if vals else 1.0


@dataclasses.dataclass
class RankChoice:
    rank: int                 # chosen rank (the largest candidate when none meets the target)
    met: bool                 # whether the chosen rank meets the target
    table: List[dict]         # per candidate: rank, mean/max cosine shift, recall, mean set size


def size_rank(ranks: Sequence[int], predict_at: Callable[[int, torch.Tensor], Sequence[np.ndarray]],
              ffn: Callable[[torch.Tensor, Sequence[np.ndarray]], np.ndarray],
              reference: Callable[[torch.Tensor], Sequence[np.ndarray]], batches: Iterable[torch.Tensor],
              max_shift: float = 0.004) -> RankChoice:
    """Smallest rank among ``ranks`` whose predicted sets keep the mean cosine
    shift of the FFN output against the ``reference`` sets at or below
    ``max_shift`` over the calibration ``batches``.

    ``predict_at(r, u)`` returns the rank-r predictor's sets for tokens u,
    ``ffn(u, sets)`` the layer output [B x d] over given sets, and
    ``reference(u)`` the reference sets (the exact ReLU mask, or the full
    predictor's)."""
    batches = list(batches)
    ranks = sorted(set(int(r) for r in ranks))
    if not ranks or not batches:
        raise ValueError("need candidate ranks and calibration tokens")
    refs = [(u, reference(u)) for u in batches]
    y_refs = [ffn(u, sets) for u, sets in refs]
    table = []
    choice = None
    for r in ranks:
        shifts, recalls, sizes = [], [], []
        for (u, ref), y_ref in zip(refs, y_refs):
            sets = predict_at(r, u)
            shifts.append(cosine_shift(ffn(u, sets), y_ref))
            recalls.append(set_recall(sets, ref))
            sizes.append(np.mean([len(s) for s in sets]))
        sh = np.concatenate(shifts)
        row = dict(rank=r, mean_shift=float(sh.mean()), max_shift=float(sh.max()), recall=float(np.mean(recalls)),
                   mean_set=float(np.mean(sizes)))
        table.append(row)
        if choice is None and row["mean_shift"] <= max_shift:
            choice = r
    return RankChoice(rank=choice if choice is not None else ranks[-1], met=choice is not None, table=table)
