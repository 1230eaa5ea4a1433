"""Build the CUDA library ``libmoe_b200.so`` in-tree for sm_100a.

Each ``csrc/*.cu`` file is compiled by nvcc (in parallel) into
``_build/*.o`` and linked into ``sparse_mixture_experts_fwd_b200/libmoe_b200.so``
with the CUDA runtime linked statically, so the library loads on a machine
without a GPU driver (the driver is reached at run time through the runtime).
The same sources are also built with ``-DMOE_CHECK_BOUNDS=1`` into
``_build/checked/`` and ``libmoe_b200_checked.so``, the bounds-checked variant
(``MOE_B200_CHECK_BOUNDS=1`` makes the Python binding load it).
``python sparse_mixture_experts_fwd_b200/build.py`` rebuilds what changed (run it
by path: importing the package itself needs the built library);
``--ptxas-info`` also writes ptxas register/spill reports to ``_build/``.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_b200.so")
LIB_CHECKED = os.path.join(PKG, "libmoe_b200_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe_b200.so")
    return path


def _deps(src: str) -> list[str]:
    return [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, ptxas_info: bool, out_dir: str = BUILD,
             defines: tuple = ()) -> tuple[str, str]:
    obj = os.path.join(out_dir, os.path.basename(src).replace(".cu", ".o"))
    cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *defines, "-c", src, "-o", obj]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if ptxas_info:
        with open(obj.replace(".o", ".ptxas.txt"), "w") as fh:
            fh.write(r.stderr)
    return obj, r.stderr


def _build_variant(out_dir: str, lib: str, defines: tuple, force: bool, ptxas_info: bool,
                   verbose: bool) -> str:
    os.makedirs(out_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    todo = [s for s in srcs
            if force or ptxas_info or _stale(os.path.join(out_dir, os.path.basename(s)[:-3] + ".o"),
                                             _deps(s))]
    if todo:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(todo))) as ex:
            for obj, log in ex.map(lambda s: _compile(s, ptxas_info, out_dir, defines), todo):
                if verbose:
                    print(f"built {obj}", file=sys.stderr)
    objs = [os.path.join(out_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if force or todo or _stale(lib, objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False,
          checked: bool = True) -> str:
    """Build libmoe_b200.so (and, unless ``checked`` is False, the bounds-checked
    libmoe_b200_checked.so); returns the default library's path."""
    _build_variant(BUILD, LIB, (), force, ptxas_info, verbose)
    if checked:
        _build_variant(os.path.join(BUILD, "checked"), LIB_CHECKED, ("-DMOE_CHECK_BOUNDS=1",),
                       force, False, verbose)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_info=a.ptxas_info, verbose=True))
