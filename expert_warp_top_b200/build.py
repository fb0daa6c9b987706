"""Build the CUDA library in-tree: libmoe_occult.so for sm_100a (B200).

    python -m expert_warp_top_b200.build [--force] [--ptxas-verbose]

Two translation units -- csrc/api.cu (inference entry points) and
csrc/api_train.cu (training entry points), each including the kernel headers it
launches -- compiled by nvcc in parallel and linked with the CUDA runtime
linked statically, so the shared object depends on no CUDA library at load
time (the driver is reached through the runtime).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libmoe_occult.so"
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not Path(cand).exists():
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe_occult.so")
    return cand


def sources() -> list[Path]:
    return (sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + sorted(CSRC.glob("*.h")) +
            [ROOT / "include" / "moe_occult.h"])


def needs_build() -> bool:
    if not LIB.exists():
        return True
    t = LIB.stat().st_mtime
    return any(p.stat().st_mtime > t for p in sources())


def build(force: bool = False, verbose_ptxas: bool = False) -> Path:
    if not force and not needs_build():
        return LIB
    from concurrent.futures import ThreadPoolExecutor
    objdir = ROOT / "_build"
    objdir.mkdir(exist_ok=True)
    flags = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
             "-I", str(ROOT / "include")]
    if verbose_ptxas:
        flags.insert(0, "-Xptxas=-v")
    units = sorted(CSRC.glob("*.cu"))
    tag = os.getpid()

    def compile_unit(src: Path):
        obj = objdir / f"{src.stem}.{tag}.o"
        res = subprocess.run([nvcc(), *flags, "-c", str(src), "-o", str(obj)],
                             capture_output=True, text=True)
        return src, obj, res

    with ThreadPoolExecutor(max_workers=len(units)) as ex:
        results = list(ex.map(compile_unit, units))
    failed = False
    for src, obj, res in results:
        if res.returncode != 0 or verbose_ptxas:
            sys.stderr.write(res.stdout + res.stderr)
        failed |= res.returncode != 0
    objs = [obj for _, obj, _ in results]
    try:
        if failed:
            raise RuntimeError(f"nvcc failed building {LIB.name}")
        tmp = LIB.with_suffix(f".so.tmp{tag}")
        res = subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", *map(str, objs),
                              "-o", str(tmp)], capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError(f"nvcc failed linking {LIB.name}")
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if obj.exists():
                obj.unlink()
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.ptxas_verbose))
