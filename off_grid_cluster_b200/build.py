"""Build libacl.so (the CUDA kernels and the C ABI) in-tree for sm_100a with nvcc.

Every .cu file is compiled to its own object in parallel (objects are reused while they are
newer than every source and header), then the objects are linked into one shared library.
`check=True` builds the check variant libacl_check.so from the same sources with
ACL_DEVICE_CHECKS defined (device-side range checks of index inputs, reported by
acl_device_check).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
OBJ = os.path.join(HERE, "_build")
SO = os.path.join(HERE, "libacl.so")
OBJ_CHECK = os.path.join(HERE, "_build_check")
SO_CHECK = os.path.join(HERE, "libacl_check.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _deps() -> list[str]:
    return sources() + _headers()


def up_to_date(check: bool = False) -> bool:
    so = SO_CHECK if check else SO
    if not os.path.exists(so):
        return False
    t = os.path.getmtime(so)
    return all(os.path.getmtime(d) <= t for d in _deps())


def _obj(src: str, check: bool) -> str:
    return os.path.join(OBJ_CHECK if check else OBJ, os.path.basename(src)[:-3] + ".o")


def _compile(nvcc: str, src: str, force: bool, verbose: bool, check: bool) -> str:
    obj = _obj(src, check)
    newest = max(os.path.getmtime(d) for d in [src, *_headers()])
    if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    tmp = obj + f".tmp{os.getpid()}"
    cmd = [nvcc, *FLAGS, *(["-DACL_DEVICE_CHECKS"] if check else []), "-I", INCLUDE, "-c", "-o", tmp, src]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, obj)
    return obj


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    so = SO_CHECK if check else SO
    if not force and not verbose and up_to_date(check):
        return so
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ_CHECK if check else OBJ, exist_ok=True)
    srcs = sources()
    with ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(nvcc, s, force, verbose, check), srcs))
    tmp = so + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH, "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, so)
    return so


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, check="--check" in sys.argv))
