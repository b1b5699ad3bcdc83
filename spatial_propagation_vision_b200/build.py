"""Build libgspn.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libgspn.so")
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
    deps += glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def build_library(force: bool = False, verbose: bool = False, jobs: int | None = None) -> str:
    """Compile every .cu under csrc/ (one object per translation unit, in
    parallel) and link them into libgspn.so; skipped when up to date."""
    if not force and not _stale():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    objdir = tempfile.mkdtemp(prefix="gspn_build_")
    try:
        cmds = []
        for src in sources():
            obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
            cmds.append(([nvcc] + NVCC_FLAGS + ["-I" + INCLUDE, "-c", "-o", obj, src], obj))
        jobs = jobs or max(1, min(len(cmds), os.cpu_count() or 1))
        procs: list[tuple[subprocess.Popen, list[str]]] = []
        pending = list(cmds)
        failed = None
        while pending or procs:
            while pending and len(procs) < jobs:
                cmd, _ = pending.pop(0)
                if verbose:
                    print(" ".join(cmd))
                procs.append((subprocess.Popen(cmd), cmd))
            p, cmd = procs.pop(0)
            if p.wait() != 0 and failed is None:
                failed = cmd
        if failed is not None:
            raise subprocess.CalledProcessError(1, failed)
        tmp = LIB + f".tmp{os.getpid()}"
        link = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp]
        link += [obj for _, obj in cmds]
        if verbose:
            print(" ".join(link))
        subprocess.check_call(link)
        os.replace(tmp, LIB)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return LIB


if __name__ == "__main__":
    print(build_library(force=True, verbose=True))
