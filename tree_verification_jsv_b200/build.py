"""Build libjsv.so in-tree with nvcc for sm_100a (no GPU needed), and its
checked twin libjsv_checked.so (-DJSV_CHECK_BOUNDS: every computed global
index is checked against its buffer and a miss is reported as
JSV_ERR_BOUNDS)."""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
SO = PKG / "libjsv.so"
SO_CHECKED = PKG / "libjsv_checked.so"
SOURCES = ["jsv_api.cu", "tree_attention.cu", "lmhead_argmax.cu", "accept_path.cu", "kv_compact.cu",
           "lmhead_noalloc.cu", "tma_host.cu", "selftest.cu",
           "tree_build.cu", "qkv_rope.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = Path(os.environ.get("CUDA_HOME", "/usr/local/cuda")) / "bin" / "nvcc"
    return str(cand) if cand.exists() else "nvcc"


def _stale(so: Path) -> bool:
    if not so.exists():
        return True
    t = so.stat().st_mtime
    deps = [CSRC / s for s in SOURCES] + list(CSRC.glob("*.cuh")) + [PKG.parent / "include" / "jsv.h"]
    return any(p.stat().st_mtime > t for p in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> Path:
    so = SO_CHECKED if checked else SO
    if not force and not _stale(so):
        return so
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           *(["-DJSV_CHECK_BOUNDS"] if checked else []),
           "-I", str(PKG.parent / "include"),
           *(str(CSRC / s) for s in SOURCES), "-o", str(so), "-lcuda"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return so


def build_all(force: bool = False, verbose: bool = False) -> list[Path]:
    """The library and its checked twin."""
    return [build(force, verbose), build(force, verbose, checked=True)]


if __name__ == "__main__":
    for p in build_all(force="--force" in sys.argv, verbose="-v" in sys.argv):
        print(p)
