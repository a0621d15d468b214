"""Compile the CPU oracle (plain C, float64) into oracle/libekv_oracle.so with gcc.

Test infrastructure: building the checker is not using it. No -ffast-math and no -march
flags, so the compiler keeps IEEE float64 semantics and the source's evaluation order.
"""
from __future__ import annotations

import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    """The oracle library; EKV_ORACLE_LIB points the loader at another build of the same
    source (the mutation tests use it to load deliberately broken copies)."""
    return os.environ.get("EKV_ORACLE_LIB") or os.path.join(_HERE, "libekv_oracle.so")


def build_oracle(force: bool = False) -> str:
    src = os.path.join(_HERE, "ekv_oracle.c")
    out = os.path.join(_HERE, "libekv_oracle.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-std=c11", "-D_DEFAULT_SOURCE", "-O2", "-fPIC", "-shared",
                           "-Wall", "-Wextra", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))
