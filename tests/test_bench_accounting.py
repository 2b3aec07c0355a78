"""bench.py's host-side accounting, on CPU: the algorithmic bytes of a step
against the published byte table of the workloads, the launch count it
claims per step against the committed ncu launch lists, and the parser of
profile summaries."""
import dataclasses
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from activation_sparse_decode_gemv_b200 import inputs  # noqa: E402

C = inputs.CONFIGS


@pytest.mark.parametrize("name,B,union,pred_mb,rows_mb,total_mb", [
    # predictor, union rows and totals per layer-step of the workloads' byte table
    ("opt7b_f16", 1, 1638, 42.0, 26.8, 68.9),
    ("opt30b_stack_f16", 1, 860, 73.5, 24.7, 98.2),
    ("llama13b_swiglu_f16", 1, 5944, 38.9, 182.6, 221.5),
    ("llama70b_swiglu_int4", 1, 14336, 75.6, 198.2, 273.9),
    ("llama70b_swiglu_int4", 32, 28672, 75.6, 396.4, 474.1),
])
def test_step_bytes_match_the_byte_table(name, B, union, pred_mb, rows_mb, total_mb):
    cfg = C[name]
    assert bench.predictor_bytes(cfg) / 1e6 == pytest.approx(pred_mb, abs=0.06)
    io = B * cfg.d * (2 + 4)  # u in (fp16), y out (fp32)
    rows = bench.step_bytes(cfg, B, union) - bench.predictor_bytes(cfg) - io
    # the ReLU layers also read the bias b1 of each row (4 B), which the table folds in
    assert rows / 1e6 == pytest.approx(rows_mb, abs=0.06)
    # the table's total counts 8 B per element of u and y (an fp32 u); the
    # library reads fp16 u, 6 B per element: 16 KB less per token at d = 8192
    table_io = 8 * B * cfg.d
    assert (bench.step_bytes(cfg, B, union) - io + table_io) / 1e6 == pytest.approx(total_mb, abs=0.15)


def test_step_bytes_small_fp32_layer():
    cfg = C["opt_tiny_f32"]
    # fp32 predictor (32 x 256 + 1024 x 32) x 4 B + bias, 8 rows of 2 x 1 KB + 4 B, u and y fp32
    assert bench.step_bytes(cfg, 1, 8) == (32 * 256 + 1024 * 32) * 4 + 4 * 1024 + 8 * (2 * 1024 + 4) + 256 * 8


def test_launch_claims_match_the_launch_lists():
    # profiles/launch_list_opt7b_f16_batch1.md: one decode_fused_kernel per step
    assert bench.kernels_per_step(C["opt7b_f16"], 1) == 1
    assert bench.kernels_per_step(C["llama70b_swiglu_int4"], 1) == 1
    # profiles/launch_list_llama13b_f16_batch4.md: the predictor kernel, the FFN kernel
    # (the compaction only when the step asks for the id lists)
    assert bench.kernels_per_step(C["llama13b_swiglu_f16"], 4) == 2
    assert bench.kernels_per_step(C["llama13b_swiglu_f16"], 4, ids=True) == 3
    # profiles/launch_list_opt7b_f16_batch8.md: the same two at batch 8
    assert bench.kernels_per_step(C["opt7b_f16"], 8) == 2
    # profiles/launch_list_llama70b_int4_batch4.md: int4 from 2 tokens on the tensor-core
    # FFN kernels, up to 8 tokens behind the batch predictor kernel
    assert bench.kernels_per_step(C["llama70b_swiglu_int4"], 4) == 4
    assert bench.kernels_per_step(C["llama70b_swiglu_int4"], 4, ids=True) == 5
    # profiles/launch_list_llama70b_int4_batch32.md: u_image, P1, P2, up/gate, down
    # (no compaction when the step asks for no id lists)
    assert bench.kernels_per_step(C["llama70b_swiglu_int4"], 32) == 5
    assert bench.kernels_per_step(C["llama70b_swiglu_int4"], 32, ids=True) == 6
    # the fp32 layer has no fused or tensor-core path
    assert bench.kernels_per_step(C["opt_tiny_f32"], 1) == 5


def test_launch_list_summaries_have_the_claimed_kernels():
    def kernel_rows(name):
        with open(os.path.join(ROOT, "profiles", name)) as fh:
            return [l for l in fh if l.startswith("| `")]
    assert len(kernel_rows("launch_list_llama13b_f16_batch4.md")) == 2
    assert len(kernel_rows("launch_list_opt7b_f16_batch8.md")) == 2
    assert len(kernel_rows("launch_list_llama70b_int4_batch4.md")) == 4
    assert len(kernel_rows("launch_list_llama70b_int4_batch32.md")) == 5


def test_profiled_traffic_parser(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "k.md").write_text(
        "# k\n\n- source_hash: `abc`\n- traffic_bytes_per_launch: `1234`\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files=None: "abc")
    assert bench.profiled_traffic("k.md") == 1234.0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files=None: "other")
    assert bench.profiled_traffic("k.md") is None       # counters of other sources
    assert bench.profiled_traffic("missing.md") is None


def test_reference_arm_line_on_cpu():
    """bench.py --impl reference times the oracle on the host and prints one
    JSON line with the contract's keys (small fp32 workload here)."""
    import json
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                          "opt_tiny_f32", "--steps", "4", "--warmup", "3"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["config"]["bias_norm"] == "pred"
    assert d["steps"] >= 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_cli_overrides():
    a = bench.parse([])
    assert a.flags == 0 and bench.config_of(a) is C["opt7b_f16"]
    from activation_sparse_decode_gemv_b200 import binding as pb
    a = bench.parse(["--hot-mode", "dense", "--flags", "1", "--bias-norm", "w1", "--config", "opt_tiny_f32"])
    assert a.flags == pb.PI_FFN_ACCUMULATE | pb.PI_FFN_HOT_DENSE
    assert bench.parse(["--hot-mode", "index"]).flags == pb.PI_FFN_HOT_INDEX
    cfg = bench.config_of(a)
    assert cfg.bias_norm == "w1" and dataclasses.replace(cfg, bias_norm="pred") == C["opt_tiny_f32"]


def test_code_tokens_ignore_comments_only():
    a = 'int f(int x) {  // sum\n  return x + 1; /* one */ }\nconst char *s = "//";'
    b = 'int f(int x) {\n  // the successor\n  return x + 1;\n}\nconst char *s = "//";'
    assert bench.code_tokens(a) == bench.code_tokens(b)
    # a changed literal or operand is a code change
    assert bench.code_tokens(a) != bench.code_tokens(a.replace("x + 1", "x + 2"))
    assert bench.code_tokens(a) != bench.code_tokens(a.replace('"//"', '"/"'))


def test_fused_profile_matches_the_kernel_code():
    """The committed DRAM-traffic summary was taken on the fused kernel's
    current code (comments aside), so the bench line can carry its traffic;
    a code change without a new capture fails here, not silently in the
    bench line."""
    t = bench.profiled_traffic("decode_fused_kernel_opt7b_f16_batch1.md")
    assert t is not None, "profiles/decode_fused_kernel_opt7b_f16_batch1.md predates the kernel code"
    assert 1.0 <= t / 69.02e6 <= 1.10  # the summary's own algorithmic bytes for that command
