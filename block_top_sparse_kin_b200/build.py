"""Build step for libkin.so (nvcc, sm_100a), kept beside the sources it builds."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libkin.so")
SOURCES = ["kin_api.cu", "kin_means.cu", "kin_select.cu", "kin_attn.cu", "kin_noalloc.cu", "kin_token.cu"]


def nvcc_command(out: str = LIB, ptxas_verbose: bool = False, defines=()) -> list:
    cmd = [
        "nvcc", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
        "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
        "-I", os.path.join(ROOT, "include"),
    ]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [f"-D{d}" for d in defines]
    cmd += [os.path.join(CSRC, s) for s in SOURCES] + ["-o", out, "-ldl"]
    return cmd


def build(verbose: bool = False, ptxas_verbose: bool = False) -> str:
    cmd = nvcc_command(ptxas_verbose=ptxas_verbose)
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_verbose=True)
