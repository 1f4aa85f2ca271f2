"""Build libcalibatt.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python -m calibrated_block_sparse_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libcalibatt.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, ptxas_verbose: bool = False, jobs: int = 4, out_path: str = None,
          defines=()) -> str:
    """Compile every csrc/*.cu and link libcalibatt.so (in-tree unless out_path)."""
    target = out_path or LIB
    if not force and not defines and out_path is None and not needs_build():
        return LIB
    cc = nvcc()
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
                    "--expt-relaxed-constexpr"]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    flags += [f"-D{d}" for d in defines]
    with tempfile.TemporaryDirectory(prefix="calibatt_build_") as tmp:
        objs = []
        procs = []
        for src in sources():
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            objs.append(obj)
            procs.append(subprocess.Popen([cc, *flags, "-c", src, "-o", obj]))
            if len(procs) >= jobs:
                if procs.pop(0).wait() != 0:
                    raise RuntimeError("nvcc failed")
        for p in procs:
            if p.wait() != 0:
                raise RuntimeError("nvcc failed")
        out = target + f".tmp{os.getpid()}"
        subprocess.check_call([cc, *ARCH, "-shared", "-o", out, *objs, "-lcudart_static", "-ldl", "-lpthread",
                               "-lrt"])
        os.replace(out, target)
    return target


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))
