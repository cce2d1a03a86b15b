"""Build the fa4q CUDA library (libfa4q.so) in-tree for sm_100a."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libfa4q.so")
SOURCES = ["api.cu", "quantize.cu", "attn_fwd.cu", "decode.cu", "decode_tc.cu", "vlines.cu", "hybrid.cu"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "fa4q.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = True) -> str:
    """Compile every CUDA source of the library for sm_100a (one nvcc process per source, in
    parallel) and link them into one shared object."""
    if not force and not _stale():
        return LIB_PATH
    from concurrent.futures import ThreadPoolExecutor
    nvcc = nvcc_path()
    flags = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC",
             "-gencode", "arch=compute_100a,code=sm_100a", "-I", INCLUDE]
    obj_dir = os.path.join(PKG_DIR, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    if verbose:
        print("[fa4q] building", os.path.relpath(LIB_PATH, ROOT), file=sys.stderr)

    def compile_one(src):
        obj = os.path.join(obj_dir, src.replace(".cu", ".o"))
        res = subprocess.run([nvcc, *flags, "-c", os.path.join(CSRC, src), "-o", obj], capture_output=True, text=True)
        return obj, res

    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        results = list(ex.map(compile_one, SOURCES))
    errors = [r.stdout + r.stderr for _, r in results if r.returncode != 0]
    if errors:
        raise RuntimeError("nvcc failed:\n" + "\n".join(errors))
    res = subprocess.run([nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", LIB_PATH + ".tmp",
                          *[o for o, _ in results]], capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv)
