"""Build libwkv.so in-tree from csrc/*.cu with nvcc for sm_100a.

    python -m wkv_recurrence_02_b200.build                  # incremental
    python -m wkv_recurrence_02_b200.build --force          # rebuild everything
    python -m wkv_recurrence_02_b200.build --debug-bounds   # bounds-checked libwkv_debug.so

Each .cu is compiled to an object under _build/ (in parallel), then linked into
wkv_recurrence_02_b200/libwkv.so with the CUDA runtime linked statically, so the
library loads on a machine without a GPU (the ABI tests use that) and finds the
driver only when a CUDA call is made.
"""
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
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libwkv.so")
# the bounds-checked debug build: every kernel checks its indices (WKV_DEBUG_BOUNDS)
BUILD_DEBUG = os.path.join(ROOT, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libwkv_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE,
              "-I", CSRC, "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _deps_newer(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    deps = [src] + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src: str, extra, verbose: bool, build_dir: str = BUILD):
    obj = os.path.join(build_dir, os.path.basename(src) + ".o")
    cmd = [nvcc()] + ARCH + NVCC_FLAGS + list(extra) + ["-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        sys.stderr.write(res.stdout + res.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, extra=(), debug_bounds: bool = False) -> str:
    """Compile every csrc/*.cu for sm_100a and link libwkv.so (or, with debug_bounds, the
    bounds-checked libwkv_debug.so); returns its path."""
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug_bounds else (BUILD, LIB)
    if debug_bounds:
        extra = tuple(extra) + ("-DWKV_DEBUG_BOUNDS",)
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    todo = [s for s in srcs
            if force or _deps_newer(os.path.join(build_dir, os.path.basename(s) + ".o"), s)]
    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(todo)))) as ex:
        list(ex.map(lambda s: _compile(s, extra, verbose, build_dir), todo))
    objs = [os.path.join(build_dir, os.path.basename(s) + ".o") for s in srcs]
    if force or todo or not os.path.exists(lib) or \
            any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", lib] + objs
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"link failed:\n{' '.join(cmd)}\n{res.stderr}")
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print -Xptxas -v (registers, spills)")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="build the bounds-checked libwkv_debug.so instead of libwkv.so")
    args = ap.parse_args()
    extra = ["-Xptxas", "-v"] if args.ptxas_info else []
    print(build(force=args.force or args.ptxas_info, verbose=args.verbose or args.ptxas_info,
                extra=extra, debug_bounds=args.debug_bounds))


if __name__ == "__main__":
    main()
