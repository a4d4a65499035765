"""Build the CPU oracle (oracle/beam_oracle.c) into oracle/_build/ with gcc.

Test infrastructure: plain C, OpenMP over tokens / rows, no BLAS.  Floating-point contraction is
off (-ffp-contract=off), so every multiply and add is rounded separately whatever the vector width;
on hosts with AVX2 the loops over independent outputs are vectorised (x86-64-v3), which changes no
value.  The library file is named after the instruction level so a build made on one host is never
loaded on a host that lacks its instructions.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "beam_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")


def _has_avx2() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("flags"):
                    flags = set(line.split(":", 1)[1].split())
                    return {"avx2", "fma", "bmi2", "movbe"} <= flags
    except OSError:
        pass
    return False


def _variant():
    if _has_avx2():
        return "v3", ["-march=x86-64-v3"]
    return "base", []


def lib_path() -> str:
    return os.path.join(OUT_DIR, f"libbeam_oracle_{_variant()[0]}.so")


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OUT_DIR, exist_ok=True)
    lib = lib_path()
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(SRC):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ftree-vectorize", "-fvect-cost-model=dynamic", "-ffp-contract=off", *_variant()[1],
           "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
