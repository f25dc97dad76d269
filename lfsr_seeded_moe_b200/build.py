"""Build libnslm.so (the CUDA library) in-tree for sm_100a with nvcc.

    python -m lfsr_seeded_moe_b200.build [--force] [--stream-source l2next|l2basis] [--bounds-check]
                                         [--table-form] [--trace]

The shared library lands in lfsr_seeded_moe_b200/_build/libnslm.so; it is
rebuilt when any source under csrc/ or include/ is newer than it.
--stream-source builds an ablation library instead, in _build/<source>/, whose
decode kernels take a block's stream bits from an L2-resident 65,536-entry
table (l2next: the 32 bits after each seed; l2basis: the 16 shifted words of
each seed) in place of the shared-memory GF(2) tables; the binding loads it
when NSLM_LIB_VARIANT names it.  --bounds-check builds _build/boundscheck/
with -DNSLM_BOUNDS_CHECK=1: every checked global access compares its index
with its extent and records the site instead of making the access (the
tests run the small parity cases on it).  --table-form builds
_build/tableform/ with -DNSLM_STACK1_F3=1: phase A of the one-token stack
takes its dot products from per-position tables of x (an ablation; slower on
B200, kept tested and measurable).  --trace builds _build/trace/ with
-DNSLM_STACK1_TRACE=1: the one-token decode kernel stamps the global timer
at its phase boundaries (`bench.py --profile anatomy` reads them).
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libnslm.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


STREAM_SOURCES = {"l2next": 1, "l2basis": 2}
VARIANT_DEFS = {"l2next": ["-DNSLM_STREAM_SOURCE=1"], "l2basis": ["-DNSLM_STREAM_SOURCE=2"],
                "boundscheck": ["-DNSLM_BOUNDS_CHECK=1"], "tableform": ["-DNSLM_STACK1_F3=1"],
                "trace": ["-DNSLM_STACK1_TRACE=1"]}


def lib_path(stream_source: str | None = None) -> str:
    return os.path.join(OUT_DIR, stream_source, "libnslm.so") if stream_source else LIB


def up_to_date(stream_source: str | None = None) -> bool:
    lib = lib_path(stream_source)
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False, extra_flags=None,
          stream_source: str | None = None) -> str:
    lib = lib_path(stream_source)
    if not force and up_to_date(stream_source):
        return lib
    out_dir = os.path.dirname(lib)
    os.makedirs(out_dir, exist_ok=True)
    defs = VARIANT_DEFS[stream_source] if stream_source else []
    jobs = []
    for src in sources():
        obj = os.path.join(out_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *defs, *(extra_flags or []), "-I", os.path.join(ROOT, "include"),
               "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        jobs.append((cmd, obj))
    # translation units compile independently: run them in parallel
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        for r in ex.map(lambda j: subprocess.run(j[0], capture_output=True, text=True), jobs):
            if r.stdout or r.stderr:
                print(r.stdout + r.stderr, file=sys.stderr, end="")
            r.check_returncode()
    objs = [o for _, o in jobs]
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]  # static cudart (nvcc default)
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    src = sys.argv[sys.argv.index("--stream-source") + 1] if "--stream-source" in sys.argv else None
    if src is not None and src not in STREAM_SOURCES:
        raise SystemExit(f"--stream-source must be one of {sorted(STREAM_SOURCES)}")
    if "--bounds-check" in sys.argv:
        src = "boundscheck"
    if "--table-form" in sys.argv:
        src = "tableform"
    if "--trace" in sys.argv:
        src = "trace"
    print(build(force="--force" in sys.argv, verbose=True, stream_source=src,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None))
