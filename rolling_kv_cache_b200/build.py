"""Build the native library librc.so in place with nvcc (sm_100a only).

Usage: python -m rolling_kv_cache_b200.build [--verbose]
The CUDA runtime is linked statically, so the library loads on a machine
without a GPU driver (host-only handles work there; device handles need a
B200).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "librc.so")
SOURCES = ["engine.cpp", "api.cu", "rope_kernels.cu", "attn_fwd.cu", "score_kernel.cu", "topc_kernel.cu",
           "rf_kernels.cu",
           "noalloc.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _newer(out, deps):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "rc.h"))
    deps.append(os.path.abspath(__file__))
    if not force and _newer(OUT, deps):
        return OUT
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O3", "-shared", "-cudart", "static",
           "-o", OUT + ".tmp"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += os.environ.get("RC_NVCC_FLAGS", "").split()  # extra -D tuning flags
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    cmd += ["-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or r.returncode:
        sys.stderr.write(r.stdout + r.stderr)
    if r.returncode:
        raise RuntimeError("nvcc failed building librc.so")
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(OUT)
