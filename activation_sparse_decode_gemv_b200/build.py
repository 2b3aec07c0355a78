"""Build libpi_ffn.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc."""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpi_ffn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr", "-Xptxas", "-v",
         "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "pi_ffn.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [NVCC] + FLAGS + ["-o", LIB + ".tmp"] + sources()
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = os.path.join(HERE, "build.log")
    with open(log, "w") as fh:
        fh.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stderr[-8000:])
        raise RuntimeError(f"nvcc failed (see {log})")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_host_sanitized(out: str) -> str:
    """The library with its HOST code built with AddressSanitizer and
    UndefinedBehaviorSanitizer into ``out`` (device code as usual), for CPU
    runs of the host-side tests; load it with the gcc sanitizer runtimes
    preloaded.  (nvcc splits -Xcompiler values at commas, hence one flag per
    sanitizer.)"""
    flags = [f for f in FLAGS if f not in ("-O3", "-Xptxas", "-v")]
    cmd = ([NVCC] + flags + ["-O1", "-g", "-Xcompiler", "-fsanitize=address", "-Xcompiler", "-fsanitize=undefined",
                             "-Xcompiler", "-fno-omit-frame-pointer", "-o", out] + sources() + ["-lasan", "-lubsan"])
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stderr[-8000:])
        raise RuntimeError("nvcc failed building the sanitized library")
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
