"""Timing of the CPU oracle on all host cores (benchmark baseline only).

TEST INFRASTRUCTURE ONLY, like the rest of this package: the benchmark's
CPU-baseline leg runs the oracle as it stands -- single-threaded C, fp64
sums -- in one process per host core, each process on whole decode tokens of
the same layer, and reports the aggregate throughput.  The layer's arrays
are shared through memory-mapped .npy files, so the processes read one copy.
Processes are started with the "spawn" method (never forked from a process
that has touched a GPU).
"""
from __future__ import annotations

import os
import time
from typing import Dict, List

import numpy as np

ARRAYS = ("w_up", "w_gate", "w_down_t", "s_up", "s_gate", "s_down_t", "b_up", "p1", "p2", "p_bias")


def save_layer(host: Dict[str, object], tokens: np.ndarray, out_dir: str) -> Dict[str, object]:
    """Write a layer's host arrays (``LayerTensors.host_arrays()``) and the
    token batch to ``out_dir``; returns the scalar fields."""
    meta = {}
    for k, v in host.items():
        if k in ARRAYS:
            if v is not None:
                np.save(os.path.join(out_dir, k + ".npy"), np.ascontiguousarray(v))
        else:
            meta[k] = v
    np.save(os.path.join(out_dir, "tokens.npy"), np.ascontiguousarray(tokens))
    return meta


def _worker(args) -> dict:
    """One process: load the shared layer, run one warm-up token, wait for
    the common start time, then run whole tokens (predictor + masked FFN over
    the predicted sets) until ``seconds`` have passed.  Returns the tokens
    run, the union size of each, and the wall-clock end."""
    out_dir, meta, first_token, seconds, t_start = args
    import oracle
    arrays = {}
    for k in ARRAYS:
        p = os.path.join(out_dir, k + ".npy")
        arrays[k] = np.load(p, mmap_mode="r") if os.path.exists(p) else None
    L = oracle.Layer(**meta, **arrays)
    toks = np.load(os.path.join(out_dir, "tokens.npy"), mmap_mode="r")
    T = toks.shape[0]

    def one(t):
        u = np.asarray(toks[t % T])
        pr = oracle.predict(L, u)
        oracle.ffn_masked(L, u, pr["idx"])
        union = np.unique(np.concatenate(pr["idx"])) if len(pr["idx"]) else np.array([], np.int64)
        return len(union)

    one(first_token)  # warm-up: page in the shared arrays
    while time.time() < t_start:
        time.sleep(0.01)
    unions: List[int] = []
    t = first_token
    while True:
        unions.append(one(t))
        t += 1
        if time.time() - t_start >= seconds:
            break
    return {"unions": unions, "end": time.time()}


def run_all_cores(out_dir: str, meta: Dict[str, object], seconds: float, workers: int,
                  start_delay: float = 20.0) -> dict:
    """Run ``workers`` spawned oracle processes concurrently for about
    ``seconds`` each.  Returns the union sizes of every token run and the
    wall time from the common start to the last process's end."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    t_start = time.time() + start_delay
    jobs = [(out_dir, meta, w * 7, seconds, t_start) for w in range(workers)]
    with ctx.Pool(workers) as pool:
        res = pool.map(_worker, jobs)
    unions = [u for r in res for u in r["unions"]]
    wall = max(r["end"] for r in res) - t_start
    return {"unions": unions, "wall": wall, "workers": workers}
