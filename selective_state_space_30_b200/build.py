"""Build the CUDA library libssmscan.so in-tree for sm_100a.

    python -m selective_state_space_30_b200.build [--force] [--debug]

The library is the product: kernels plus the C ABI declared in
include/ssm_scan.h.  Each translation unit compiles in parallel.  --debug builds
libssmscan_debug.so from the same sources with SSM_DEBUG defined: the scan
kernels then check their indices against the buffers they touch and record
SSM_ERR_BOUNDS in the device status word instead of making a bad access.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libssmscan.so")
LIB_DEBUG = os.path.join(HERE, "libssmscan_debug.so")
BUILD_DIR = os.path.join(HERE, "_build")
BUILD_DIR_DEBUG = os.path.join(HERE, "_build_debug")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v", f"-I{INCLUDE}"]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src: str, extra, build_dir=BUILD_DIR) -> str:
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    log = obj + ".ptxas.txt"
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    with open(log, "w") as f:
        f.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{res.stderr[-4000:]}")
    return obj


def _stale(lib, outputs_newer_than):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in outputs_newer_than)


def build(force: bool = False, extra=(), debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    build_dir = BUILD_DIR_DEBUG if debug else BUILD_DIR
    extra = list(extra) + (["-DSSM_DEBUG"] if debug else [])
    deps = sources() + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)] + \
        [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    if not force and not _stale(lib, deps):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, build_dir), srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stderr[-4000:]}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, debug="--debug" in sys.argv))
