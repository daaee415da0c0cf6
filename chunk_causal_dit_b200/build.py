"""Build libwf.so in-tree with nvcc for sm_100a (B200).

    python -m chunk_causal_dit_b200.build [--force] [--verbose] [--check]

--check builds the debug variant libwf_check.so (compiled with -DWF_CHECK: the
kernels' computed global indices are bounds-checked, a failure is reported by
wf_sync_status as WF_ERR_BOUNDS instead of trapping).  The binding loads it
instead of libwf.so when WF_LIB_VARIANT=check is set in the environment.

The library is written next to this file (chunk_causal_dit_b200/libwf.so) so
that it travels with the source tree; the CUDA runtime is linked statically,
and the driver's tensor-map encoder is fetched at run time, so the library has
no link-time dependency on libcuda and loads on machines without a GPU.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libwf.so")
LIB_CHECK = os.path.join(HERE, "libwf_check.so")
SOURCES = ["wf_api.cu", "append_kernel.cu", "attn_kernel.cu", "attn_pair_kernel.cu",
           "quant_fp8_kernel.cu", "noalloc.cu", "gemm_kernel.cu", "ln_kernel.cu", "vae_kernel.cu"]
HEADERS = ["sm100.cuh", "wf_internal.h", "exp2_poly.h", "wf_check.cuh", "fp8_rule.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "wf.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    lib = LIB_CHECK if check else LIB
    if not force and up_to_date(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc, *NVCC_FLAGS, *(["-DWF_CHECK"] if check else []), "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--check", action="store_true", help="build the WF_CHECK debug variant")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, check=a.check))


if __name__ == "__main__":
    main()
