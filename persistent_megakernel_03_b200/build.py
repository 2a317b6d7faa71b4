"""Builds libmk.so (the CUDA path) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmk.so")
# The debug-bounds build: the same sources with MK_DEBUG_BOUNDS, whose tasks
# check every access and report a violation through mk_status.
LIB_DEBUG = os.path.join(HERE, "libmk_debug.so")
SOURCES = ["plan.cpp", "kernel.cu", "step_bf16_d128.cu", "step_bf16_d64.cu", "step_fp8_d128.cu",
           "step_fp8_d64.cu", "api.cu", "attention.cu", "prefill.cu",
           "prefill_mk.cu", "flash_attn.cu"]
HEADERS = ["mk_internal.h", "plan.h", "ptx.cuh", "attn_math.cuh", "tc.cuh", "prefill.h",
           "step_kernel.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "mk.h"))
    return files


def is_fresh(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra=(), debug_bounds: bool = False) -> str:
    """Compiles every source to an object in parallel (one nvcc per file),
    then links the shared library (libmk.so, or libmk_debug.so with
    debug_bounds); skipped when the library is newer than every source and
    header."""
    out = LIB_DEBUG if debug_bounds else LIB
    if debug_bounds:
        extra = (*extra, "-DMK_DEBUG_BOUNDS")
    if not force and is_fresh(out):
        return out
    from concurrent.futures import ThreadPoolExecutor
    import tempfile
    nvcc = os.environ.get("NVCC", "nvcc")
    common = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
              "-I", os.path.join(ROOT, "include"), *extra]
    if verbose:
        common.insert(0, "-Xptxas=-v")
    with tempfile.TemporaryDirectory(prefix="mk_build_") as tmpdir:
        def compile_one(src):
            obj = os.path.join(tmpdir, os.path.splitext(src)[0] + ".o")
            r = subprocess.run([nvcc, *common, "-c", os.path.join(CSRC, src), "-o", obj],
                               cwd=CSRC, capture_output=True, text=True)
            return src, obj, r
        with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
            results = list(ex.map(compile_one, SOURCES))
        failed = [r for r in results if r[2].returncode != 0]
        for src, _, r in results:
            if r.returncode != 0 or verbose:
                sys.stderr.write(f"--- {src}\n" + r.stdout + r.stderr)
        if failed:
            raise RuntimeError("nvcc failed building libmk.so: " + ", ".join(f[0] for f in failed))
        tmp = out + f".tmp{os.getpid()}"
        r = subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *[o for _, o, _ in results]],
                           cwd=CSRC, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed linking libmk.so")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug_bounds="--debug-bounds" in sys.argv))
