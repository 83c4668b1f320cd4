"""Builds libnvfp4.so (the CUDA library behind include/nvfp4.h) in-tree with nvcc for sm_100a,
and its debug twin libnvfp4_checked.so: the same sources with -DNVFP4_BOUNDS_CHECK, whose
kernels check every global access against its buffer's extent (include/nvfp4.h,
nvfp4_bounds_checked).  The translation units of both are compiled in parallel.

The quantizer translation unit is compiled with -fmad=false (no contracted multiply-adds)
and without fast math, so its FP32 arithmetic is exactly the recipe's.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libnvfp4.so")
CHECKED_LIB = os.path.join(PKG, "libnvfp4_checked.so")
BUILD_DIR = os.path.join(PKG, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
          "--expt-relaxed-constexpr"]
UNITS = {
    "api.cu": [],
    "quantize.cu": ["-fmad=false"],
    "gemm.cu": [],
    "noalloc.cu": [],
}
# library path, object folder and extra defines of each variant
VARIANTS = {
    "release": (LIB, os.path.join(BUILD_DIR, "release"), []),
    "checked": (CHECKED_LIB, os.path.join(BUILD_DIR, "checked"), ["-DNVFP4_BOUNDS_CHECK"]),
}


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _sources():
    out = []
    for name in os.listdir(CSRC):
        if name.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, name))
    out.append(os.path.join(INCLUDE, "nvfp4.h"))
    out.append(os.path.abspath(__file__))  # a change of flags rebuilds too
    return out


def up_to_date(variant: str = "release") -> bool:
    lib = VARIANTS[variant][0]
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in _sources())


def build(force: bool = False, verbose: bool = False,
          variants=("release", "checked")) -> str:
    """Compile the requested variants (all units at once) and link each; returns the release
    library's path."""
    todo = [v for v in variants if force or not up_to_date(v)]
    nvcc = _nvcc()
    jobs = []
    for v in todo:
        _, obj_dir, defines = VARIANTS[v]
        os.makedirs(obj_dir, exist_ok=True)
        for unit, extra in UNITS.items():
            obj = os.path.join(obj_dir, unit.replace(".cu", ".o"))
            cmd = [nvcc, *ARCH, *COMMON, *defines, *extra, "-c", os.path.join(CSRC, unit),
                   "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), file=sys.stderr)
            jobs.append((v, obj, cmd, subprocess.Popen(cmd)))
    failed = [" ".join(cmd) for _, _, cmd, proc in jobs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    for v in todo:
        lib, _, _ = VARIANTS[v]
        objs = [obj for w, obj, _, _ in jobs if w == v]
        subprocess.run([nvcc, *ARCH, "-shared", "-o", lib, *objs], check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
