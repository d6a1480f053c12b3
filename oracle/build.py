"""Compile the C oracle with gcc (test infrastructure; no CUDA involved).

    python -m oracle.build          # builds oracle/_liboracle.so
"""
from __future__ import annotations

import os
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))


def oracle_lib_path(mutant: int = 0) -> str:
    name = "_liboracle.so" if mutant == 0 else f"_liboracle_mutant{mutant}.so"
    return os.path.join(_HERE, name)


def build_oracle(mutant: int = 0) -> str:
    src = os.path.join(_HERE, "sdpa_oracle.c")
    out = oracle_lib_path(mutant)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    if mutant:
        cmd.insert(1, f"-DORACLE_MUTANT={int(mutant)}")
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(int(sys.argv[1]) if len(sys.argv) > 1 else 0))
