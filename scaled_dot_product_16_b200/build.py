"""Build libattn.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m scaled_dot_product_16_b200.build            # incremental
    python -m scaled_dot_product_16_b200.build --force    # rebuild everything

Each .cu file in csrc/ is compiled to an object under _build/ (skipped when newer than its
sources), then linked into scaled_dot_product_16_b200/libattn.so. A second copy built with the
test flags (STALL_FLAGS) becomes libattn_stalltest.so, which only the timeout test loads. No GPU
is needed.
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libattn.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


# The test build: identical sources, with the attention kernel's pipeline waits bounded at 1 ms
# and one extra wait on a barrier that nothing arrives on, so that a GPU test sees that wait run
# out and the kernel report ATTN_ERR_TIMEOUT, drain its own work and exit (drains keep 200 ms).
STALL_LIB = os.path.join(PKG, "libattn_stalltest.so")
STALL_FLAGS = ["-DSDPA_TEST_STALL=1", "-DSDPA_PIPE_WAIT_NS=1000000ull"]


def _build_lib(lib: str, objdir: str, extra, force: bool, verbose: bool) -> str:
    os.makedirs(objdir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    hdr_time = _newest(headers) if headers else 0.0
    objs = []
    for src in sources:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), hdr_time)):
            continue
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < _newest(objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-ldl",
                        "-lpthread", "-lrt"], check=True)
        os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    return _build_lib(LIB, BUILD, [], force, verbose)


def build_stall_test(force: bool = False) -> str:
    return _build_lib(STALL_LIB, os.path.join(BUILD, "stalltest"), STALL_FLAGS, force, False)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas resource usage")
    args = ap.parse_args(argv)
    print(build(force=args.force, verbose=args.verbose))
    print(build_stall_test(force=args.force))
    return 0


if __name__ == "__main__":
    sys.exit(main())
