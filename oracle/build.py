"""Build the fp64 CPU oracle (test infrastructure only) into oracle/liboracle.so.

Plain gcc, no fast-math, no FMA contraction, OpenMP across independent units.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "wkv_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(src: str = SRC, out: str = LIB, quiet: bool = True) -> str:
    """Compile `src` into the shared library `out` and return its path."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
           src, "-o", out, "-lm"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + " ".join(cmd) + "\n" + res.stderr)
    if not quiet and res.stderr:
        sys.stderr.write(res.stderr)
    return out


def up_to_date(src: str = SRC, out: str = LIB) -> bool:
    return os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src)


if __name__ == "__main__":
    print(build(quiet=False))
