"""Builds libveda.so in-tree for sm_100a with nvcc (``python -m learned_block_sparse_tile_b200.build``)."""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libveda.so")

SOURCES = ["veda_api.cu", "veda_plan.cpp", "veda_score_noalloc.cu"]
HEADERS = ["veda_internal.h", "ptx.cuh", "gather.cuh", "score.cuh", "select.cuh", "attend.cuh", "attend_pair.cuh",
           "quant.cuh"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out=LIB, extra=()):
    return [nvcc_path(), "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-ffp-contract=off",
            "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), "-I", CSRC, *extra,
            "-o", out] + [os.path.join(CSRC, s) for s in SOURCES]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "veda.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, verbose=False, extra=()):
    """Compiles the library when a source is newer than it (or when ``force``). Returns its path."""
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = command(tmp, extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    build(force=True, verbose=True, extra=[a for a in args if a.startswith("-")])
