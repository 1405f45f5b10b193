"""Build libkdn.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension).

    python -m delta_rule_recurrent_scan_b200.build [--force]

The library lands in ``delta_rule_recurrent_scan_b200/lib/libkdn.so``; it is
rebuilt when any source under ``csrc/`` or ``include/`` is newer.
"""

from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libkdn.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]
# IEEE single precision everywhere except the chunked tensor-core kernel, whose operands are
# well-scaled (no denormals matter) and whose reciprocals and divisions sit on serial chains.
IEEE_FLAGS = ["-ftz=false", "-prec-div=true", "-prec-sqrt=true"]
PER_FILE_FLAGS = {name: ["-ftz=true", "-prec-div=false", "-prec-sqrt=false"] for name in ("chunk_scan.cu", "chunk_scan_ws.cu", "pside.cu", "hola_tc.cu")}


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    obj_dir = os.path.join(LIB_DIR, "obj")
    os.makedirs(obj_dir, exist_ok=True)
    cmds, objs = [], []
    for src in sources():
        name = os.path.basename(src)
        obj = os.path.join(obj_dir, name + ".o")
        cmds.append([_nvcc(), *NVCC_FLAGS, *PER_FILE_FLAGS.get(name, IEEE_FLAGS), "-I", INCLUDE, "-c", src, "-o", obj])
        objs.append(obj)

    def compile_one(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)

    workers = max(1, min(len(cmds), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=workers) as pool:
        list(pool.map(compile_one, cmds))
    tmp = LIB + ".tmp"
    link = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
            "-Xcompiler", "-fPIC", "-o", tmp, *objs]
    if verbose:
        print(" ".join(link), flush=True)
    subprocess.run(link, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
