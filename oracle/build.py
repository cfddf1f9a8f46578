"""Compile the float64 delta-rule oracle (``dr_oracle.c``) into a shared library.

Test infrastructure only: the tests, the smoke check and the benchmark's
CPU-baseline leg load the result; the CUDA library never does.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dr_oracle.c")
LIB = os.path.join(HERE, "libdr_oracle.so")


def build(force: bool = False, out: str = LIB, extra_flags=(), src: str = SRC) -> str:
    """Build ``libdr_oracle.so`` next to its source (or ``src`` into ``out``); return its path."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    # -ffp-contract=off: every product and sum rounds as written (no fused multiply-add).
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           *extra_flags, src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
