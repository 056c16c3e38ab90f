"""Compile the CUDA kernels and the C ABI into block_sparse_long_compress_b200/libqsa.so.

sm_100a only (tcgen05 / TMEM / TMA).  The CUDA runtime is linked
statically; the driver's cuTensorMapEncodeTiled is reached through the
runtime's driver entry-point query, so the library needs no libcuda at
link time and loads on a machine without a GPU.
"""
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "qsa_lib.cu")
LIB = os.path.join(HERE, "libqsa.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include", "qsa.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--cudart", "static",
]


def _sources():
    out = [INCLUDE]
    for f in sorted(os.listdir(SRC_DIR)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(SRC_DIR, f))
    return out


# The prefill kernel moves registers between its warpgroups (setmaxnreg):
# its split is sized for this many registers per thread at launch (the
# launch bounds' ceiling for 384 threads).  A kernel launched with fewer
# would wait forever in setmaxnreg.inc, so the build refuses it.
PREFILL_LAUNCH_REGS = 168


def _check_registers(ptxas_log: str) -> None:
    entry = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and "sparse_attn_prefill_kernel" in entry:
            if int(m.group(1)) != PREFILL_LAUNCH_REGS:
                raise RuntimeError(
                    f"{entry} launches with {m.group(1)} registers per thread; its setmaxnreg "
                    f"split assumes {PREFILL_LAUNCH_REGS}")
            entry = None


def build(force: bool = False, verbose: bool = False) -> str:
    """Build libqsa.so if missing or older than any source; return its path."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t for s in _sources()):
            return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    if not os.path.exists(nvcc) and os.path.exists("/usr/local/cuda/bin/nvcc"):
        nvcc = "/usr/local/cuda/bin/nvcc"
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, "-Xptxas=-v", *NVCC_FLAGS, "-o", tmp, MAIN]
    r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)
    if verbose or r.returncode != 0:
        sys.stdout.write(r.stdout)
    if r.returncode != 0:
        raise subprocess.CalledProcessError(r.returncode, cmd)
    try:
        _check_registers(r.stdout)
    except RuntimeError:
        os.remove(tmp)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
