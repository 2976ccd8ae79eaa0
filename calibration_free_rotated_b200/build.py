"""Builds liborbitquant.so in-tree with nvcc for sm_100a.

Usage:  python -m calibration_free_rotated_b200.build   (or build() from Python)

The library links the CUDA runtime statically and nothing else from CUDA, so it
loads on a machine without a GPU driver (host planning still works there);
driver entry points it needs are resolved at run time through the runtime.
"""

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "liborbitquant.so")
SOURCES = ["oq_host.cpp", "oq_rotq.cu", "oq_rotq_cfg0.cu", "oq_rotq_cfg1.cu", "oq_rotq_cfg2.cu",
           "oq_rotq_cfg0_np.cu", "oq_rotq_cfg1_np.cu", "oq_rotq_cfg2_np.cu", "oq_rotq_composed.cu", "oq_cbgemm.cu",
           "oq_noalloc.cu", "oq_flatness.cu"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build liborbitquant.so")
    return exe


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(os.path.dirname(HERE), "include", "orbitquant.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compiles every source into one shared library; returns its path."""
    if not force and not _stale():
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    nvcc = _nvcc()
    jobs = []
    for src in SOURCES:
        obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
        cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(os.path.dirname(HERE), "include"),
               "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        jobs.append((cmd, obj))
    # the translation units are independent: compile them side by side
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        for f in [ex.submit(subprocess.run, cmd, check=True) for cmd, _ in jobs]:
            f.result()
    objs = [obj for _, obj in jobs]
    tmp = LIB + ".tmp"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static", "-shared",
           "-Xcompiler", "-fPIC", *objs, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
