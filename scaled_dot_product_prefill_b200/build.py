"""Build libattn_b200.so (the CUDA and C++ sources under csrc/) for sm_100a with nvcc.

Each translation unit is compiled to an object under ``_build/`` (in
parallel, skipped when up to date) and linked into
``scaled_dot_product_prefill_b200/libattn_b200.so`` next to this file.
The CUDA runtime is linked statically and the driver's tensor-map encoder
is looked up at run time, so the library loads on machines without a GPU
driver (where every compute call then fails with ATTN_ERR_CUDA).
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
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libattn_b200.so")

SOURCES = ["attn_api.cu", "prefill_sm100.cu", "prefill_f32.cu", "decode_paged.cu", "kv_append.cu", "page_pool.cpp"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# Host code is built without exceptions and uses only the C library and
# pthreads, so the .so needs no C++ runtime: a late dlopen of libstdc++ can
# fail for want of static TLS when the host process has not loaded it yet.
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fno-exceptions",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]
LINK_FLAGS = ["-Xlinker", "--as-needed", "-lpthread"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libattn_b200.so")


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return hs


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, extra):
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    path = os.path.join(CSRC, src)
    if not _stale(obj, [path, __file__] + _headers()) and not extra:
        return obj, None
    cmd = [nvcc()] + ARCH + FLAGS + list(extra) + ["-c", path, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        return obj, f"{' '.join(cmd)}\n{r.stdout}\n{r.stderr}"
    return obj, (r.stdout + r.stderr) if extra else None


def build(verbose: bool = False, extra=()) -> str:
    """Compile and link the library; returns its path.  Raises on compiler errors."""
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(lambda s: _compile(s, extra), SOURCES))
    errs = [msg for _, msg in results if msg and "error" in msg.lower()]
    if errs:
        raise RuntimeError("nvcc failed:\n" + "\n".join(errs))
    if verbose:
        for _, msg in results:
            if msg:
                print(msg)
    objs = [o for o, _ in results]
    if _stale(LIB, objs) or extra:
        cmd = [nvcc()] + ARCH + ["-shared", "-o", LIB] + objs + LINK_FLAGS
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    extra = sys.argv[1:]
    print(build(verbose=True, extra=extra))
