"""Compile the PSA CUDA library (libpsa.so) for sm_100a, in-tree.

Usage: python -m level_sparse_attention_b200.build [--debug]

--debug builds libpsa_debug.so, the same sources with PSA_DEBUG defined
(device-side bounds checks of the work lists).
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = ["pyramid.cu", "mask.cu", "score_tc.cu", "attn_simt.cu", "attn_tc.cu", "psa_api.cu",
           "psa_noalloc.cu", "psa_selftest.cu", "psa_host.cu", "bwd_aux.cu", "attn_bwd_simt.cu",
           "attn_bwd_tc.cu"]
LIB = os.path.join(HERE, "libpsa.so")
DEBUG_LIB = os.path.join(HERE, "libpsa_debug.so")


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC"]


def build(verbose: bool = False, debug: bool = False) -> str:
    """Compile every source to an object in _build/ (in parallel), then link
    libpsa.so (libpsa_debug.so with ``debug``).  Skipped when the library is
    newer than every source."""
    from concurrent.futures import ThreadPoolExecutor
    lib_path = DEBUG_LIB if debug else LIB
    srcs = [os.path.join(HERE, "csrc", s) for s in SOURCES]
    deps = srcs + [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))
                   if f.endswith(".cuh")] + [os.path.join(ROOT, "include", "psa.h")]
    if os.path.exists(lib_path) and all(os.path.getmtime(lib_path) >= os.path.getmtime(d)
                                        for d in deps):
        return lib_path
    out_dir = os.path.join(ROOT, "_build", "debug" if debug else "release")
    os.makedirs(out_dir, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include")] + (["-DPSA_DEBUG"] if debug else [])

    def compile_one(src):
        obj = os.path.join(out_dir, os.path.basename(src) + ".o")
        cmd = [nvcc()] + FLAGS + inc + ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        return obj

    with ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib_path + ".tmp"
    cmd = [nvcc()] + FLAGS + ["-shared", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(verbose=True, debug="--debug" in sys.argv[1:]))
