"""Build ``libwq.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m gemm_wq_gemv_b200.build [--force] [--verbose] [--checks]``.
The library carries sm_100a machine code only (``-gencode arch=compute_100a,
code=sm_100a``); it links the CUDA runtime statically and needs no CUDA
driver library at link time.  ``--checks`` builds the checked library
(``libwq_checked.so``, compiled with ``WQ_CHECKS``: every kernel checks the
index of each access it computes itself and records a failed check instead of
making the access; see ``wq_checked_build`` in include/wq.h).  The sources
compile in parallel.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
CSRC = PKG / "csrc"
ROOT = PKG.parent
LIB = PKG / "libwq.so"
LIB_CHECKED = PKG / "libwq_checked.so"
BUILD = ROOT / "_build"
SOURCES = ["wq_abi.cu", "wq_host.cu", "wq_pack.cu", "wq_gemv.cu", "wq_gemv_lean.cu", "wq_gemm.cu",
           "wq_noalloc.cu", "wq_mse.cu", "wq_gptq.cu", "wq_selftest.cu"]
HEADERS = ["wq_internal.h", "wq_ptx.cuh", "wq_dequant.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        p = Path(cand) / "bin" / "nvcc"
        if cand and p.exists():
            return str(p)
    found = shutil.which("nvcc")
    if not found:
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libwq.so")
    return found


def _stale(lib: Path = LIB) -> bool:
    if not lib.exists():
        return True
    t = lib.stat().st_mtime
    deps = [CSRC / s for s in SOURCES + HEADERS] + [ROOT / "include" / "wq.h", Path(__file__)]
    return any(d.stat().st_mtime > t for d in deps)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> Path:
    lib = LIB_CHECKED if checks else LIB
    if not force and not _stale(lib):
        return lib
    out = BUILD / ("checked" if checks else "normal")
    out.mkdir(parents=True, exist_ok=True)
    cc = nvcc()
    common = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "--expt-relaxed-constexpr", "-I", str(ROOT / "include")]
    if checks:
        common += ["-DWQ_CHECKS"]
    if verbose:
        common += ["-Xptxas", "-v"]
    objs = [str(out / (Path(src).stem + ".o")) for src in SOURCES]
    jobs = [subprocess.Popen([cc, *common, "-c", str(CSRC / src), "-o", obj]) for src, obj in zip(SOURCES, objs)]
    failed = [src for src, j in zip(SOURCES, jobs) if j.wait() != 0]
    if failed:
        raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
    tmp = lib.with_suffix(f".so.tmp{os.getpid()}")
    subprocess.run([cc, *ARCH, "-shared", "-o", str(tmp), *objs], check=True)
    os.replace(tmp, lib)
    return lib


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--checks", action="store_true", help="build the checked library (WQ_CHECKS)")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, checks=a.checks))
    return 0


if __name__ == "__main__":
    sys.exit(main())
