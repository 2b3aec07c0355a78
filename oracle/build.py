"""Compile the CPU oracle (plain C, gcc) into oracle/libpi_oracle.so.

The oracle is test infrastructure: the test suite, the smoke check and the
benchmark's CPU-baseline leg load it; the CUDA library never does.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pi_oracle.c")
LIB = os.path.join(HERE, "libpi_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    # -O2 without -ffast-math keeps IEEE semantics; -ffp-contract=off forbids
    # fused multiply-add so every product and sum is rounded as written.
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_sanitized(out: str) -> str:
    """The same oracle built with AddressSanitizer and UndefinedBehaviorSanitizer
    (halting on the first report) into ``out``; load it with the gcc sanitizer
    runtimes preloaded."""
    cmd = ["gcc", "-std=c11", "-O1", "-g", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fsanitize=address", "-fsanitize=undefined", "-fno-sanitize-recover=undefined",
           "-fno-omit-frame-pointer", "-o", out, SRC, "-lm"]
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
