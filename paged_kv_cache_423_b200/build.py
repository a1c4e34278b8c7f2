"""Build libpkv.so in-tree with nvcc for sm_100a.

``python -m paged_kv_cache_423_b200.build`` (or ``build_library()``) compiles every
source under ``csrc/`` into ``_build/*.o`` in parallel and links
``paged_kv_cache_423_b200/libpkv.so``.  The CUDA runtime is linked statically, so the
library loads on machines without a GPU (the NVIDIA driver is only needed once a call
touches the device).  ptxas register/shared-memory reports go to
``_build/ptxas.log``.  Rebuilds only when a source or header is newer than the
library.

``variant="depth1"`` builds ``libpkv_depth1.so`` (objects under ``_build/depth1``) with the
CUDA-core decode kernel's per-warp copy ring at one stage, so every copy waits for the
previous stage's compute; a test compares it bit for bit with the default build.

``variant="shortwait"`` builds ``libpkv_shortwait.so`` whose CUDA-core decode and prefill
kernels give up a pipeline wait after one poll instead of one second, so an ordinary launch takes its expiry path (flag PKV_DEV_TIMEOUT, let copies land,
wait for MMAs, free tensor memory, return); a test checks the flag and that the context
stays usable.  No wait is removed and the drains keep their one-second limit.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpkv.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
              "--expt-relaxed-constexpr", "-Xcompiler", "-fvisibility=hidden"]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-fvisibility=hidden"]
VARIANTS = {"depth1": ["-DPKV_SIMT_STAGES=1", "-DPKV_SIMT_STAGES8=1"],
            "shortwait": ["-DPKV_SHORT_WAITS"]}


def lib_path(variant: str | None = None) -> str:
    return LIB if variant is None else os.path.join(PKG, f"libpkv_{variant}.so")


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libpkv.so")
    return path


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    files.append(os.path.abspath(__file__))
    return files


def is_stale(variant: str | None = None) -> bool:
    lib = lib_path(variant)
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def _compile(src: str, build_dir: str = BUILD, extra_defs=()) -> tuple[str, str]:
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    inc = ["-I", INCLUDE, "-I", CSRC]
    # Exported symbols carry default visibility through the header's extern "C" block.
    defs = ["-DPKV_BUILD", *extra_defs]
    if src.endswith(".cu"):
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *inc, *defs, "-c", src, "-o", obj]
    else:
        cmd = [nvcc(), "-x", "c++", *ARCH, "-O2", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler",
               "-fvisibility=hidden", *inc, *defs, "-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"compiling {os.path.basename(src)} failed:\n{' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    return obj, res.stderr


def build_library(force: bool = False, verbose: bool = False, variant: str | None = None) -> str:
    lib = lib_path(variant)
    if not force and not is_stale(variant):
        return lib
    build_dir = BUILD if variant is None else os.path.join(BUILD, variant)
    extra = () if variant is None else VARIANTS[variant]
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda src: _compile(src, build_dir, extra), srcs))
    with open(os.path.join(build_dir, "ptxas.log"), "w") as f:
        for (obj, log), src in zip(results, srcs):
            f.write(f"==== {os.path.basename(src)}\n{log}\n")
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *[o for o, _ in results], "-cudart", "static"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"linking libpkv.so failed:\n{' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, lib)
    if verbose:
        print(f"built {lib}")
    return lib


if __name__ == "__main__":
    v = sys.argv[sys.argv.index("--variant") + 1] if "--variant" in sys.argv else None
    build_library(force="--force" in sys.argv, verbose=True, variant=v)
