#!/usr/bin/env python
"""Benchmark of the sparse-FFN decode hot path on B200.

One step = one full pass of the decode path over one token batch of one FFN
layer: predictor (h = P1 u, s = P2 h + b, threshold), compaction of the active
ids, gathered up/gate rows with the activation, gathered down-projection rows,
reduction.  Default workload: the OPT-7B-shaped fp16 ReLU layer (d = 4096,
f = 16384, rank-1024 predictor, mean firing rate 10%, hot prefix 20%) at
batch 1.  Steps rotate through 8 independently seeded layer replicas (2.5 GB,
far above the 126 MB L2) and 32 seeded tokens, so weights come from HBM.

Metric: achieved HBM GB/s over the bytes the step touches (predictor weights
and bias + up/gate and down rows of the predicted union + token in / y out),
with us per layer alongside.  Timed
with CUDA events around graph replays; N > 1 GPUs run independent replicas
(weak scaling, no collective on the data path) and the time is the maximum
over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

from activation_sparse_decode_gemv_b200 import inputs

def kernels_per_step(cfg, B, ids=False):
    """Launches of the library's kernels per decode step (the library's
    dispatch, see pi_decode_ffn in include/pi_ffn.h): batch 1 with fp16 / int4
    weights runs as one persistent fused kernel; fp16 batches of 2..8 run two
    (the persistent predictor kernel, the persistent FFN kernel); int4
    batches of 2..8 run four (that predictor kernel, then the tensor-core
    token image, up/gate and down GEMMs); int4 batches of 9..32 and fp16
    batches of 9..32 run five on the tensor-core path (token image, two
    predictor GEMMs, up/gate and down GEMMs); the compaction adds one when
    the call asks for the id lists (``ids``); anything else runs five
    CUDA-core kernels (predictor stage 1, stage 2, compaction, gather,
    reduction)."""
    if B == 1 and cfg.wtype != "f32" and cfg.r <= 1024 and cfg.d <= 8192:
        return 1
    pred_batch = (2 <= B <= 8 and cfg.wtype != "f32" and cfg.r % 64 == 0 and cfg.r <= 1024
                  and cfg.d % 64 == 0 and cfg.d <= 8192 and cfg.r <= 8 * 148)
    tc_min = 2 if cfg.wtype == "int4g32" else 9
    if tc_min <= B <= 32 and cfg.wtype != "f32" and (cfg.wtype != "int4g32" or cfg.d % 256 == 0):
        n = 4 if pred_batch else 5
        return n + 1 if ids else n
    if pred_batch and cfg.wtype == "f16" and cfg.f <= 32768:
        return 3 if ids else 2
    return 5


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=4000)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="opt7b_f16")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--replicas", type=int, default=8)
    ap.add_argument("--tokens", type=int, default=32)
    ap.add_argument("--flags", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-workers", type=int, default=64,
                    help="oracle processes of the all-core CPU baseline (at most the host's cores; 0 skips it)")
    ap.add_argument("--stack-config", default="opt30b_stack_f16",
                    help="stacked workload timed as the line's 'stack' object at batch 1 ('none' skips it)")
    ap.add_argument("--stack-steps", type=int, default=200)
    ap.add_argument("--batch-configs", default="opt7b_f16:8,llama13b_swiglu_f16:4,llama70b_swiglu_int4:4,"
                    "llama70b_swiglu_int4:32",
                    help="config:batch pairs timed as the line's 'batches' objects ('none' skips them)")
    ap.add_argument("--batch-steps", type=int, default=400)
    ap.add_argument("--json-out", default=None)
    ap.add_argument("--stack", action="store_true",
                    help="time pi_decode_ffn_stack through all layers of a stacked config (tokens/s)")
    ap.add_argument("--hot-mode", default="auto", choices=sorted(HOT_MODE_FLAGS),
                    help="read the hot prefix densely, by index, or as the library decides (adds to --flags)")
    ap.add_argument("--rank", type=int, default=0,
                    help="cut every layer's predictor to its leading RANK components (0: the config's rank)")
    ap.add_argument("--bias-norm", default=None, choices=["pred", "w1"],
                    help="predictor bias scale of the generated layers (default: the config's)")
    args = ap.parse_args(argv)
    args.flags |= HOT_MODE_FLAGS[args.hot_mode]
    return args


# library flag bits (include/pi_ffn.h): PI_FFN_HOT_DENSE = 2, PI_FFN_HOT_INDEX = 4
HOT_MODE_FLAGS = {"auto": 0, "dense": 2, "index": 4}


def config_of(args) -> inputs.Config:
    """The workload of --config, with the --bias-norm override."""
    cfg = inputs.CONFIGS[args.config]
    return cfg.scaled(bias_norm=args.bias_norm) if args.bias_norm else cfg


RAMP_SECONDS = 0.03


def clock_ramp(work) -> float:
    """Untimed replays of ``work`` for RAMP_SECONDS before the warm-up steps,
    so that a short timed run starts at the clocks of a busy GPU (a timed
    region of a few hundred microseconds right after the idle setup would
    otherwise include the ramp).  Returns the seconds spent."""
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < RAMP_SECONDS:
        work()
        torch.cuda.synchronize()
    return time.perf_counter() - t0


def sized(args, lt):
    """The layer with its predictor cut to ``--rank`` leading components
    (the predictor sizing of the calibration module), or as generated."""
    if not args.rank or args.rank == lt.r:
        return lt
    from activation_sparse_decode_gemv_b200 import calibrate
    return calibrate.truncate_predictor(lt, args.rank)


# ----------------------------------------------------------------------------- distributed plumbing

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(bytes_per_rank: float, seconds_per_rank: float, world: int):
    """Whole-job GB/s: all ranks' bytes over the slowest rank's time."""
    t = max_over_ranks(seconds_per_rank, world)
    b = sum_over_ranks(bytes_per_rank, world)
    return b / t / 1e9, t


# ----------------------------------------------------------------------------- bytes of a step

def row_bytes(cfg: inputs.Config) -> int:
    if cfg.wtype == "f32":
        return cfg.d * 4
    if cfg.wtype == "f16":
        return cfg.d * 2
    return cfg.d // 2 + (cfg.d // 32) * 2


def predictor_bytes(cfg: inputs.Config) -> int:
    e = 4 if cfg.wtype == "f32" else 2
    return (cfg.r * cfg.d + cfg.f * cfg.r) * e + 4 * cfg.f


def step_bytes(cfg: inputs.Config, B: int, n_union: int) -> int:
    """Bytes of one step: predictor factors and bias, the up (and gate) and
    down rows of the union of the predicted sets (plus the ReLU bias), u in and
    y out."""
    n_mat = 3 if cfg.act == "swiglu" else 2
    ue = 4 if cfg.wtype == "f32" else 2
    bias = 4 if cfg.act == "relu" else 0
    return (predictor_bytes(cfg) + n_union * (n_mat * row_bytes(cfg) + bias) + B * cfg.d * ue + B * cfg.d * 4)


# ----------------------------------------------------------------------------- profile summaries

# device sources the fused batch-1 kernel is compiled from
FUSED_SOURCES = ("pi_fused.cuh", "pi_device.cuh")


def code_tokens(src: str) -> str:
    """C/CUDA source with its comments removed and its whitespace collapsed
    (string and character literals kept as they are): edits to comments or
    layout leave it unchanged, any edit to the code does not."""
    import re
    tok = re.compile(r'"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|//[^\n]*|/\*.*?\*/|\s+|[^"\'/\s]+|/', re.S)
    out = []
    for m in tok.finditer(src):
        t = m.group(0)
        if t.startswith("//") or t.startswith("/*") or t.isspace():
            if out and out[-1] != " ":
                out.append(" ")
        else:
            out.append(t)
    return "".join(out).strip()


def kernel_source_hash(files=FUSED_SOURCES) -> str:
    """Hash of the code (comments and layout excluded) of the CUDA sources a
    kernel is built from; a profile summary's counters apply only to the
    kernel built from the code it records."""
    import hashlib
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "activation_sparse_decode_gemv_b200", "csrc", name), encoding="utf-8") as fh:
            h.update(code_tokens(fh.read()).encode())
            h.update(b"\0")
    return h.hexdigest()[:16]


def profiled_traffic(summary: str):
    """DRAM bytes per launch (read + write) from a profiles/ summary, or None
    when the summary is missing or was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as fh:
        for line in fh:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_hash") != kernel_source_hash():
        return None
    try:
        return float(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.file.flush()
        rows = []
        with open(self.file.name) as fh:
            for line in fh:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_run(layer_host: inputs.LayerTensors, cfg, u_host: torch.Tensor, seconds: float, max_steps: int):
    """Time the oracle (as it stands, one host thread) on whole tokens until the
    time budget is spent.  Returns (steps, seconds, bytes)."""
    import oracle
    L = oracle.Layer(**layer_host.host_arrays())
    n, t_tot, b_tot = 0, 0.0, 0
    T = u_host.shape[0]
    while n < max_steps:
        u = u_host[n % T].numpy()
        t0 = time.perf_counter()
        pr = oracle.predict(L, u)
        y = oracle.ffn_masked(L, u, pr["idx"])
        dt = time.perf_counter() - t0
        union = np.unique(np.concatenate(pr["idx"])) if len(pr["idx"]) else np.array([], np.int64)
        t_tot += dt
        b_tot += step_bytes(cfg, u.shape[0], len(union))
        n += 1
        if t_tot >= seconds:
            break
    return n, t_tot, b_tot


# ----------------------------------------------------------------------------- main

def bench_reference(args, world, rank):
    if rank != 0:
        return None
    cfg = config_of(args)
    lt = sized(args, inputs.make_layer(cfg, 0, seed=1000, device="cuda" if torch.cuda.is_available() else "cpu")).to("cpu")
    cfg = lt.cfg
    toks = torch.stack([inputs.layer_input(cfg, inputs.make_tokens(cfg, t, args.batch, seed=1000))
                        for t in range(args.tokens)])
    # warm-up: the requested count of whole tokens, at most 3 (one oracle token
    # at the OPT-7B shape takes about half a second)
    wu = max(1, min(args.warmup, 3))
    oracle_run(lt, cfg, toks, float("inf"), wu)
    n, sec, nbytes = oracle_run(lt, cfg, toks, args.ref_seconds, args.steps)
    v = nbytes / sec / 1e9
    line = {"metric": "sparse-FFN achieved HBM GB/s of touched rows (batch-1 decode)", "value": v, "unit": "GB/s",
            "impl": "reference", "n_gpus": args.gpus, "steps": n, "warmup": wu, "ms_per_step": sec / n * 1e3,
            "us_per_layer": sec / n * 1e6, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{cfg.name} single FFN layer d={cfg.d} f={cfg.f} r={cfg.r} {cfg.wtype} "
                                   f"batch {args.batch}", "batch": args.batch, "bias_norm": cfg.bias_norm},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{n} whole tokens of replica 0 (time-bounded at {args.ref_seconds:.0f} s)"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def bench_ours(args, world, rank, local):
    from activation_sparse_decode_gemv_b200 import binding as pb
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    pb.lib()
    dev = torch.device("cuda", local)
    cfg = config_of(args)
    B, R, T = args.batch, args.replicas, args.tokens
    seed = 1000 + rank
    layers = [sized(args, inputs.make_layer(cfg, r, seed=seed, device=dev)) for r in range(R)]
    cfg = layers[0].cfg
    handles = [pb.FfnLayer.from_tensors(lt) for lt in layers]
    ws = pb.make_workspace(handles, B, dev)
    toks_host = torch.stack([inputs.layer_input(cfg, inputs.make_tokens(cfg, t, B, seed=seed)) for t in range(T)])
    toks = toks_host.to(dev)
    y = torch.zeros((B, cfg.d), device=dev)
    stream = torch.cuda.Stream(dev)

    # bytes of every (replica, token) pair, from the library's own sets (untimed)
    pair_bytes = {}
    idx = torch.empty((B, cfg.f), dtype=torch.int32, device=dev)
    cnt = torch.empty((B,), dtype=torch.int32, device=dev)
    for r in range(R):
        lt = layers[r]
        for t in range(T):
            pb.pi_decode_ffn(handles[r], toks[t], y, ws, idx=idx, count=cnt, flags=args.flags)
            torch.cuda.synchronize()
            c = cnt.cpu().tolist()
            sets = [idx[b, :c[b]].long() for b in range(B)]
            union = torch.unique(torch.cat(sets)) if sum(c) else torch.empty(0, dtype=torch.long, device=dev)
            pair_bytes[(r, t)] = step_bytes(cfg, B, len(union))
    assert pb.pi_get_device_status(ws) == 0

    # graphs: one of S = lcm(R, T) consecutive steps (the schedule's period),
    # plus one graph of the first n steps for a remainder n, so that a run of
    # K steps is K // S replays of the period and at most one more launch, and
    # consecutive steps overlap through programmatic dependent launch
    S = int(np.lcm(R, T))
    sched = [(j % R, j % T) for j in range(S)]

    def step(j):
        r, t = sched[j]
        pb.pi_decode_ffn(handles[r], toks[t], y, ws, flags=args.flags, stream=stream)

    with torch.cuda.stream(stream):
        for j in range(S):  # eager warm-up before capture
            step(j)
    stream.synchronize()

    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j in range(n):
                step(j)
        return g

    period = capture(S)
    heads = {n: capture(n) for n in {args.warmup % S, args.steps % S} if n}

    def run(nsteps):
        with torch.cuda.stream(stream):
            for _ in range(nsteps // S):
                period.replay()
            if nsteps % S:
                heads[nsteps % S].replay()

    # every graph the timed run launches has been launched once before: a
    # graph's first launch uploads it to the device
    with torch.cuda.stream(stream):
        for g in heads.values():
            g.replay()
    ramp_s = clock_ramp(lambda: run(S))
    run(args.warmup)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        run(args.steps)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    sec = ev0.elapsed_time(ev1) / 1e3
    assert pb.pi_get_device_status(ws) == 0
    nbytes = sum(pair_bytes[sched[j % S]] for j in range(args.steps))
    gbs, tmax = aggregate(nbytes, sec, world)
    us_layer = tmax / args.steps * 1e6

    # End to end through the public call with pinned host buffers: every step
    # copies its token in (H2D) and its y out (D2H).  The copies run on a
    # second stream with double-buffered u and y, so step j+1's upload and
    # step j-1's download overlap step j's decode, and the step sequence is a
    # CUDA graph (the host issues nothing per step).
    h_in = toks_host.pin_memory()
    E = S
    h_out = torch.empty((E, B, cfg.d), dtype=torch.float32).pin_memory()
    u_buf = [torch.empty_like(toks[0]) for _ in range(2)]
    y_buf = [torch.empty_like(y) for _ in range(2)]
    cstream = torch.cuda.Stream(dev)

    def e2e_sequence():
        ev_in = [torch.cuda.Event() for _ in range(E)]
        ev_y = [torch.cuda.Event() for _ in range(E)]
        ev_out = [torch.cuda.Event() for _ in range(E)]
        cstream.wait_stream(stream)
        with torch.cuda.stream(cstream):
            u_buf[0].copy_(h_in[sched[0][1]], non_blocking=True)
            ev_in[0].record(cstream)
        for j in range(E):
            r, _ = sched[j]
            if j + 1 < E:  # upload the next token (its buffer was last read by step j-1)
                with torch.cuda.stream(cstream):
                    u_buf[(j + 1) % 2].copy_(h_in[sched[j + 1][1]], non_blocking=True)
                    ev_in[j + 1].record(cstream)
            stream.wait_event(ev_in[j])
            if j >= 2:  # y buffer of step j-2 downloaded
                stream.wait_event(ev_out[j - 2])
            pb.pi_decode_ffn(handles[r], u_buf[j % 2], y_buf[j % 2], ws, flags=args.flags, stream=stream)
            ev_y[j].record(stream)
            with torch.cuda.stream(cstream):
                cstream.wait_event(ev_y[j])
                h_out[j].copy_(y_buf[j % 2], non_blocking=True)
                ev_out[j].record(cstream)
        stream.wait_stream(cstream)

    with torch.cuda.stream(stream):
        e2e_sequence()  # eager warm-up
    torch.cuda.synchronize()
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        e2e_sequence()
    reps = max(1, args.e2e_steps // E)
    n_e2e = reps * E
    with torch.cuda.stream(stream):
        ge.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            ge.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_sec = e0.elapsed_time(e1) / 1e3
    e2e_bytes = sum(pair_bytes[sched[j % S]] for j in range(n_e2e))
    e2e_gbs, _ = aggregate(e2e_bytes, e2e_sec, world)
    # the downloaded y must equal the device result of the same step
    with torch.cuda.stream(stream):
        pb.pi_decode_ffn(handles[sched[E - 1][0]], toks[sched[E - 1][1]], y, ws, flags=args.flags, stream=stream)
    torch.cuda.synchronize()
    assert torch.equal(h_out[E - 1], y.cpu()), "end-to-end output differs from the device result"

    peaks = {}
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        peaks = json.load(open(pp))
    peak = peaks.get("hbm_gbs", 6650.0)
    per_gpu = gbs / world
    line = {
        "metric": "sparse-FFN achieved HBM GB/s of touched rows (batch-1 decode)",
        "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tmax / args.steps * 1e3, "us_per_layer": us_layer,
        "ffn_layer_tokens_per_s": B * args.steps / tmax * world,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "weights": cfg.wtype, "data": "synthetic",
        "config": {"workload": f"{cfg.name}: single FFN layer d={cfg.d} f={cfg.f} r={cfg.r} {cfg.act} "
                               f"{cfg.wtype} weights, batch {B}, mean firing rate {cfg.mean_p}",
                   "batch": B, "d_model": cfg.d, "d_ffn": cfg.f, "rank": cfg.r, "replicas": R, "tokens": T,
                   "l2": f"{R} rotating seeded replicas ({sum(l.nbytes() for l in layers) / 1e9:.1f} GB) > L2",
                   "bytes_per_step": nbytes / args.steps, "parallelism": f"replicas x{world}",
                   "bias_norm": cfg.bias_norm, "hot_mode": args.hot_mode,
                   "outputs": "y per step; the timed calls pass no idx/count, so the ascending global id list "
                              "(step 2's optional output) is not written inside the timed region",
                   "graphs": f"one CUDA graph per {S} consecutive steps (remainder: one graph of the first "
                             f"steps), consecutive launches overlapping through programmatic dependent launch",
                   "untimed_before_warmup": f"each graph launched once, then {ramp_s * 1e3:.0f} ms of replays "
                                            f"of the {S}-step graph (clock ramp)"},
        "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": peak, "unit": "GB/s", "frac": per_gpu / peak,
                     "traffic": (profiled_traffic(f"decode_fused_kernel_{cfg.name}_batch{B}.md")
                                 if kernels_per_step(cfg, B) == 1 and not args.rank else None),
                     "algorithmic_bytes_per_launch": nbytes / args.steps,
                     "kernel": ("decode_fused_kernel (the whole step is one launch)" if kernels_per_step(cfg, B) == 1
                                else f"whole decode step ({kernels_per_step(cfg, B)} kernels)"),
                     "peak_source": "measured" if "hbm_gbs" in peaks else "fallback"},
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": int(toks[0].numel() * toks.element_size()),
                "d2h_bytes_per_step": int(y.numel() * 4), "steps": n_e2e,
                "us_per_layer": e2e_sec / n_e2e * 1e6,
                "copies": "pinned host buffers; H2D and D2H every step on a second stream, double-buffered, "
                          "overlapping the neighbouring steps' decode; graph-captured step sequence"},
        "gpu_launches": kernels_per_step(cfg, B) * args.steps,
        "clocks": clk.summary(),
    }
    if args.stack_config != "none":
        line["stack"] = stack_summary(args, world, rank, local)
    if args.batch_configs != "none":
        line["batches"] = [batch_summary(args, world, rank, local, spec) for spec in args.batch_configs.split(",")]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = layers[0].to("cpu")
        del layers, handles
        n, csec, cbytes = oracle_run(host, cfg, toks_host, args.cpu_seconds, 10 ** 9)
        line["cpu_baseline"] = {"value": cbytes / csec / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} whole tokens of replica 0, one host thread",
                                "us_per_layer": csec / n * 1e6}
        workers = min(args.cpu_workers, os.cpu_count() or 1)
        if workers > 1:
            line["cpu_baseline_all_cores"] = oracle_all_cores(host, cfg, toks_host, args.cpu_seconds, workers)
    return line


def oracle_all_cores(host, cfg, toks_host, seconds, workers):
    """The oracle as it stands, one spawned process per core, each on whole
    tokens of the same layer (shared through memory-mapped files), for about
    ``seconds``; aggregate GB/s = all processes' bytes over the wall time."""
    import shutil
    from oracle import timing
    d = tempfile.mkdtemp(prefix="pi_oracle_")
    try:
        meta = timing.save_layer(host.host_arrays(), toks_host.numpy(), d)
        res = timing.run_all_cores(d, meta, seconds, workers)
    finally:
        shutil.rmtree(d, ignore_errors=True)
    B = toks_host.shape[1]
    nbytes = sum(step_bytes(cfg, B, u) for u in res["unions"])
    n = len(res["unions"])
    return {"value": nbytes / res["wall"] / 1e9, "unit": "GB/s", "cores": res["workers"],
            "host_cpu_count": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} whole tokens of replica 0 over {res['wall']:.1f} s, one single-threaded oracle "
                      f"process per core ({res['workers']} processes)",
            "us_per_layer_per_process": res["wall"] * res["workers"] / n * 1e6}


def stack_summary(args, world, rank, local):
    """Batch-1 FFN-stack decode of ``--stack-config`` (every layer, RMS norm,
    predictor, sparse FFN, residual add), for the main line's 'stack' object."""
    import copy
    a = copy.copy(args)
    a.config, a.batch, a.tokens = args.stack_config, 1, 4
    a.steps, a.warmup = args.stack_steps, max(3, args.stack_steps // 10)
    st = bench_stack(a, world, rank, local)
    torch.cuda.empty_cache()
    return {"workload": st["config"]["workload"], "tokens_per_s": st["value"], "us_per_layer": st["us_per_layer"],
            "steps": st["steps"], "warmup": st["warmup"], "layers": st["config"]["layers"],
            "bytes_per_token": st["config"]["bytes_per_step"], "roofline": st["roofline"],
            "gpu_launches_per_token": st["gpu_launches_per_step"], "clocks": st["clocks"],
            "generation_s": st["config"]["generation_s"]}


def batch_summary(args, world, rank, local, spec):
    """One multi-token single-layer configuration (``config:batch``), timed
    like the main line (rotating replicas larger than L2, CUDA graphs, CUDA
    events), for the line's 'batches' objects."""
    import copy
    name, b = spec.split(":")
    a = copy.copy(args)
    a.config, a.batch, a.replicas, a.tokens = name, int(b), 4, 8
    a.steps, a.warmup, a.e2e_steps = args.batch_steps, max(3, args.batch_steps // 10), 16
    a.stack_config, a.batch_configs, a.no_cpu_baseline, a.cpu_workers, a.rank = "none", "none", True, 0, 0
    ln = bench_ours(a, world, rank, local)
    torch.cuda.empty_cache()
    return {"workload": ln["config"]["workload"], "batch": a.batch, "us_per_layer": ln["us_per_layer"],
            "value": ln["value"], "unit": ln["unit"], "steps": ln["steps"], "warmup": ln["warmup"],
            "bytes_per_step": ln["config"]["bytes_per_step"], "roofline": ln["roofline"],
            "gpu_launches_per_step": ln["gpu_launches"] // ln["steps"], "clocks": ln["clocks"]}


def bench_stack(args, world, rank, local):
    """FFN-stack decode: every layer of a stacked config (RMS norm, predictor,
    sparse FFN, residual add), one token batch per pass, timed with CUDA
    events around graph replays.  Attention is not part of the path."""
    from activation_sparse_decode_gemv_b200 import binding as pb
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    pb.lib()
    dev = torch.device("cuda", local)
    cfg = config_of(args)
    assert cfg.stacked, f"{cfg.name} is not a stacked config"
    B, L, T = args.batch, cfg.n_layers, args.tokens
    seed = 3000 + rank
    t0 = time.perf_counter()
    layers = [sized(args, inputs.make_layer(cfg, l, seed=seed, device=dev)) for l in range(L)]
    cfg = layers[0].cfg
    gen_s = time.perf_counter() - t0
    handles = [pb.FfnLayer.from_tensors(lt) for lt in layers]
    ws = pb.make_workspace(handles, B, dev)
    xs = [inputs.make_tokens(cfg, t, B, seed=seed).to(dev) for t in range(T)]
    x = torch.empty_like(xs[0])
    stream = torch.cuda.Stream(dev)
    # bytes per pass from the stack's own traces (untimed)
    idx = torch.empty((L, B, cfg.f), dtype=torch.int32, device=dev)
    cnt = torch.empty((L, B), dtype=torch.int32, device=dev)
    tok_bytes = []
    for t in range(T):
        x.copy_(xs[t])
        pb.pi_decode_ffn_stack(handles, x, ws, idx_trace=idx, count_trace=cnt, flags=args.flags)
        torch.cuda.synchronize()
        c = cnt.cpu()
        nb = 0
        for l in range(L):
            sets = [idx[l, b, :int(c[l, b])].long() for b in range(B)]
            union = torch.unique(torch.cat(sets)) if int(c[l].sum()) else torch.empty(0, dtype=torch.long)
            nb += step_bytes(cfg, B, len(union))
        tok_bytes.append(nb)
    assert pb.pi_get_device_status(ws) == 0
    graphs = []
    for t in range(T):
        with torch.cuda.stream(stream):
            x.copy_(xs[t])
            pb.pi_decode_ffn_stack(handles, x, ws, flags=args.flags, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            x.copy_(xs[t])
            pb.pi_decode_ffn_stack(handles, x, ws, flags=args.flags, stream=stream)
        graphs.append(g)

    def run(n):
        with torch.cuda.stream(stream):
            for j in range(n):
                graphs[j % T].replay()

    # every graph the timed run launches has been launched once before: a
    # graph's first launch uploads it to the device
    run(T)
    clock_ramp(lambda: run(T))
    run(args.warmup)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev0.record(stream)
        run(args.steps)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    sec = ev0.elapsed_time(ev1) / 1e3
    assert pb.pi_get_device_status(ws) == 0
    nbytes = sum(tok_bytes[j % T] for j in range(args.steps))
    gbs, tmax = aggregate(nbytes, sec, world)
    peaks = {}
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        peaks = json.load(open(pp))
    peak = peaks.get("hbm_gbs", 6650.0)
    return {
        "metric": "FFN-stack decode tokens/s (attention excluded)",
        "value": B * args.steps / tmax * world, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tmax / args.steps * 1e3, "us_per_layer": tmax / args.steps / L * 1e6,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "weights": cfg.wtype,
        "data": "synthetic",
        "config": {"workload": f"{cfg.name}: {L}-layer FFN stack d={cfg.d} f={cfg.f} r={cfg.r} {cfg.act} "
                               f"{cfg.wtype} weights, batch {B}",
                   "batch": B, "layers": L, "tokens": T, "weights_gb": sum(l.nbytes() for l in layers) / 1e9,
                   "bytes_per_step": nbytes / args.steps, "generation_s": gen_s,
                   "bias_norm": cfg.bias_norm, "hot_mode": args.hot_mode},
        "roofline": {"bound": "hbm", "achieved": gbs / world, "peak": peak, "unit": "GB/s",
                     "frac": gbs / world / peak, "peak_source": "measured" if "hbm_gbs" in peaks else "fallback"},
        "gpu_launches_per_step": L * (kernels_per_step(cfg, B) + (0 if kernels_per_step(cfg, B) == 1 else 1)),
        "clocks": clk.summary(),
    }


def main(argv=None):
    args = parse(argv)
    world, rank, local = dist_init()
    try:
        if args.impl == "reference":
            line = bench_reference(args, world, rank)
        elif args.stack:
            line = bench_stack(args, world, rank, local)
        else:
            line = bench_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            s = json.dumps(line)
            print(s, flush=True)
            if args.json_out:
                with open(args.json_out, "w") as fh:
                    fh.write(s + "\n")
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
