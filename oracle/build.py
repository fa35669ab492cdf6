"""Compile the CPU oracle (test infrastructure) into oracle/_build/libqsa_oracle.so."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qsa_oracle.cpp")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libqsa_oracle.so")


def build(force: bool = False, sanitize: bool = False) -> str:
    """Build the oracle library (or an ASan/UBSan variant) and return its path."""
    os.makedirs(OUT_DIR, exist_ok=True)
    out = LIB if not sanitize else os.path.join(OUT_DIR, "libqsa_oracle_san.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-fopenmp",
           SRC, "-o", out + ".tmp"]
    if sanitize:
        cmd[3:3] = ["-fsanitize=address,undefined", "-fno-omit-frame-pointer", "-g"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True, sanitize="--sanitize" in sys.argv))
