"""Build libs2attn.so (the C-ABI library) in-tree with nvcc for sm_100a, and
libs2attn_debug.so, the same sources with the kernels' bounds checks compiled
in (-DS2_DEBUG_BOUNDS).

    python -m shifted_sparse_attention_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libs2attn.so"
DEBUG_LIB = PKG / "libs2attn_debug.so"
SOURCES = ["s2attn_api.cu", "s2_fwd.cu", "s2_bwd.cu", "s2_adj.cu", "s2_docs.cu", "s2_gap.cu", "s2_rope.cu", "s2_sp.cu", "s2attn_noalloc.cu"]
HEADERS = ["s2_index.cuh", "sm100_ptx.cuh", "s2_kernels.h", "s2_debug.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
]


def _stale(lib: Path) -> bool:
    if not lib.exists():
        return True
    t = lib.stat().st_mtime
    deps = [CSRC / s for s in SOURCES + HEADERS] + [ROOT / "include" / "s2attn.h", Path(__file__)]
    return any(d.stat().st_mtime > t for d in deps)


def _build_one(lib: Path, sub: str, extra: list[str], verbose: bool) -> None:
    build_dir = PKG / "_build" / sub
    build_dir.mkdir(parents=True, exist_ok=True)
    objs = []
    procs = []
    for src in SOURCES:
        obj = build_dir / (Path(src).stem + ".o")
        cmd = [NVCC, *FLAGS, *extra, "-I", str(ROOT / "include"), "-c", str(CSRC / src), "-o", str(obj)]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
        objs.append(str(obj))
    failed = False
    for cmd, pr in procs:
        out, _ = pr.communicate()
        if out and (verbose or pr.returncode):
            sys.stderr.write(out)
        if pr.returncode:
            sys.stderr.write("FAILED: %s\n" % " ".join(cmd))
            failed = True
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = lib.with_suffix(".so.tmp%d" % os.getpid())
    subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", str(tmp)])
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> Path:
    """Both libraries; returns the path of the normal one."""
    if force or _stale(LIB):
        _build_one(LIB, "release", [], verbose)
    if force or _stale(DEBUG_LIB):
        _build_one(DEBUG_LIB, "debug", ["-DS2_DEBUG_BOUNDS"], verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
