"""Host sanitizers on CPU: the oracle and the C-ABI library's host code built
with AddressSanitizer and UndefinedBehaviorSanitizer (halting on the first
report), each driven by its own host-side tests in a child process with the
gcc sanitizer runtimes preloaded.  A planted out-of-bounds read and a planted
signed overflow (in a throw-away C file, on the CPU) show that the harness
reports what it should."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _runtime(name):
    p = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


ASAN, UBSAN = _runtime("libasan.so"), _runtime("libubsan.so")
pytestmark = pytest.mark.skipif(not (ASAN and UBSAN), reason="gcc sanitizer runtimes not installed")


def _env(**extra):
    env = dict(os.environ)
    env.update(LD_PRELOAD=f"{ASAN}:{UBSAN}", ASAN_OPTIONS="detect_leaks=0:protect_shadow_gap=0",
               UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1", PYTHONPATH=ROOT, CUDA_VISIBLE_DEVICES="")
    env.update(extra)
    return env


def _pytest(files, **extra):
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu"] + \
          [os.path.join(ROOT, "tests", f) for f in files]
    return subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT, env=_env(**extra))


def _clean(out):
    text = out.stdout + out.stderr
    return out.returncode == 0 and "ERROR: AddressSanitizer" not in text and "runtime error:" not in text


def test_harness_reports_planted_errors(tmp_path):
    src = tmp_path / "planted.c"
    src.write_text(
        "#include <stdlib.h>\n"
        "int oob(int i) { int *a = malloc(4 * sizeof(int)); int v = a[i]; free(a); return v; }\n"
        "int ovf(int x) { return x + 1; }\n")
    lib = tmp_path / "libplanted.so"
    subprocess.check_call(["gcc", "-O0", "-g", "-fPIC", "-shared", "-fsanitize=address", "-fsanitize=undefined",
                           "-fno-sanitize-recover=undefined", "-o", str(lib), str(src)])
    for call, marker in (("oob(4)", "AddressSanitizer"), ("ovf(2147483647)", "runtime error")):
        code = f"import ctypes; ctypes.CDLL({str(lib)!r}).{call}"
        out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120, env=_env())
        assert out.returncode != 0 and marker in out.stderr, (call, out.returncode, out.stderr[-500:])


def test_oracle_under_asan_ubsan(tmp_path):
    sys.path.insert(0, ROOT)
    from oracle import build
    lib = build.build_sanitized(str(tmp_path / "libpi_oracle_san.so"))
    out = _pytest(["test_oracle_pins.py", "test_calibrate.py"], PI_ORACLE_LIB=lib)
    assert _clean(out), (out.stdout + out.stderr)[-3000:]


def test_abi_host_code_under_asan_ubsan(tmp_path):
    sys.path.insert(0, ROOT)
    from activation_sparse_decode_gemv_b200 import build
    lib = build.build_host_sanitized(str(tmp_path / "libpi_ffn_san.so"))
    out = _pytest(["test_abi_host.py", "test_binding_checks.py"], PI_FFN_LIB=lib)
    assert _clean(out), (out.stdout + out.stderr)[-3000:]
    assert "passed" in out.stdout
