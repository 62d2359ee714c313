"""Builds libgtr_gla.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m recurrent_vision_backbone_key_b200.build [--force] [--checked]``.
Each .cu file under csrc/ is compiled to an object in parallel, then all are
linked into ``recurrent_vision_backbone_key_b200/libgtr_gla.so`` with a
static CUDA runtime.  ``--checked`` also builds the bounds-checked debug
library ``libgtr_gla_checked.so`` (the same sources with -DGTR_BOUNDS_CHECK).
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libgtr_gla.so")
OBJ_DIR_CHECKED = os.path.join(PKG, "_build_checked")
LIB_CHECKED = os.path.join(PKG, "libgtr_gla_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_dep() -> float:
    deps = glob.glob(os.path.join(CSRC, "*")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max(os.path.getmtime(p) for p in deps)


def _compile(src: str, extra: list[str], obj_dir: str = OBJ_DIR) -> str:
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip():
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    """Compile every csrc/*.cu and link libgtr_gla.so (or, with checked=True,
    libgtr_gla_checked.so with -DGTR_BOUNDS_CHECK); returns its path."""
    lib, obj_dir = (LIB_CHECKED, OBJ_DIR_CHECKED) if checked else (LIB, OBJ_DIR)
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _newest_dep():
        return lib
    os.makedirs(obj_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    extra = (["-Xptxas", "-v"] if verbose_ptxas else []) + (["-DGTR_BOUNDS_CHECK"] if checked else [])
    with cf.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, obj_dir), srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-lrt", "-lpthread", "-ldl"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas-v" in sys.argv))
    if "--checked" in sys.argv:
        print(build(force="--force" in sys.argv, checked=True))
