"""Build the native library ``libsparse_attn.so`` in place with nvcc for sm_100a.

The library is the product's compute path: every step of mask construction
and attention runs in its CUDA kernels. It links the CUDA runtime statically
and resolves the driver's tensor-map encoder at run time, so loading it needs
no GPU (the ABI tests load it on CPU-only machines).

``build(debug=True)`` builds ``libsparse_attn_debug.so`` from the same sources
with SA_DEBUG_CHECKS defined: indices that come from data (mask lists, slot
maps, union lists) are tested before they address memory and a failure sets
the bounds flag of the status word (``tests/test_gpu_debug_build.py`` runs it).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsparse_attn.so")
LIB_DEBUG = os.path.join(HERE, "libsparse_attn_debug.so")
SOURCES = ["sa_api.cu", "sa_mask.cu", "sa_attn.cu", "sa_fg.cu", "sa_noalloc.cu", "sa_selftest.cu",
           "sa_profile.cu", "sa_quant.cu"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
              "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static"]


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(HERE, "..", "include", "sparse_attn.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force=False, verbose=False, debug=False):
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    objs = []
    for src in SOURCES:
        obj = os.path.join(CSRC, "_build_debug" if debug else "_build", src.replace(".cu", ".o"))
        os.makedirs(os.path.dirname(obj), exist_ok=True)
        cmd = [nvcc, *NVCC_FLAGS, *(["-DSA_DEBUG_CHECKS"] if debug else []),
               "-I", os.path.join(HERE, "..", "include"), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = lib + ".tmp"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
           "-Xcompiler", "-fPIC", *objs, "-o", tmp, "-lrt", "-ldl", "-lpthread"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv)
