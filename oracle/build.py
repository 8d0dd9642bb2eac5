"""Compile the float64 oracle (oracle.c) into a shared library with gcc.

Test infrastructure: the result is loaded only by the tests, the package smoke
check and the bench's CPU-baseline leg.  ``mutation`` > 0 builds a variant with
one planted mistake, used to show that the oracle's pins catch such mistakes.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")


def lib_path(mutation: int = 0, out_dir: str | None = None) -> str:
    name = "liboracle.so" if mutation == 0 else f"liboracle_mut{mutation}.so"
    return os.path.join(out_dir or HERE, name)


def build(mutation: int = 0, out_dir: str | None = None, force: bool = False) -> str:
    out = lib_path(mutation, out_dir)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    # -ffp-contract=off: every product and sum is rounded as written, in double.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           f"-DORACLE_MUTATION={int(mutation)}", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(int(sys.argv[1]) if len(sys.argv) > 1 else 0, force=True))
