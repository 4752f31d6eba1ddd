"""Builds libinfini_attn.so in-tree with nvcc for sm_100a.

Run ``python -m compressive_memory_transformer_sm_b200.build`` (or call
``build()``).  The library links the CUDA runtime statically so that it does
not depend on which libcudart another framework in the process has loaded.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libinfini_attn.so")
ARCH = "-gencode=arch=compute_100a,code=sm_100a"


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libinfini_attn")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(ROOT, "include", "infini_attn.h"), __file__]
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = LIB + ".tmp"
    cmd = [nvcc_path(), ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include"),
           "-o", tmp, os.path.join(CSRC, "infini_attn.cu")]
    extra = os.environ.get("INFINI_NVCC_FLAGS", "").split()
    cmd[1:1] = extra + ["-Xptxas=-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed with exit code {res.returncode}")
    if verbose:
        print(res.stdout + res.stderr, flush=True)
    check_register_split(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


def check_register_split(ptxas_log: str, kernel: str = "attn_tc_kernel", want: int = 168) -> None:
    """The attention kernel redistributes registers between warpgroups (setmaxnreg)
    assuming it was launched with exactly `want` registers per thread; any other
    allocation could make a register increase wait forever, so refuse to build."""
    lines = ptxas_log.splitlines()
    checked = 0
    for i, line in enumerate(lines):
        if "Compiling entry function" in line and kernel in line:  # every instantiation
            for nxt in lines[i + 1:i + 6]:
                if "Used" in nxt and "registers" in nxt:
                    used = int(nxt.split("Used")[1].split("registers")[0])
                    if used != want:
                        raise RuntimeError(f"{kernel} uses {used} registers per thread, its register split "
                                           f"assumes {want}: refusing to build")
                    checked += 1
                    break
    if checked == 0:
        raise RuntimeError(f"ptxas report for {kernel} not found: cannot verify its register split")


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
