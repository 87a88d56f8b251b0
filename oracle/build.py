"""Build the CPU oracle (plain C) into oracle/libmoe_oracle.so.

Test infrastructure: compiled by the package build step so that the tests,
the smoke check and the benchmark's CPU baseline can load it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libmoe_oracle.so")
SRC = [os.path.join(HERE, "moe_oracle.c")]


def build(force: bool = False) -> str:
    deps = SRC + [os.path.join(HERE, "moe_oracle.h")]
    if not force and os.path.exists(LIB):
        if os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in deps):
            return LIB
    # -ffp-contract=off: every float operation of the quantiser is a separate
    # IEEE rounding, as written.
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-o", LIB] + SRC + ["-lm"]
    subprocess.check_call(cmd)
    return LIB


def build_mutant(n: int, out_dir: str) -> str:
    """Oracle with planted mistake number n (see ORC_MUTANT in moe_oracle.c).

    Used only by the test that checks the oracle's pins catch such mistakes."""
    out = os.path.join(out_dir, "libmoe_oracle_mut%d.so" % n)
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-DORC_MUTANT=%d" % n, "-o", out] + SRC + ["-lm"]
    subprocess.check_call(cmd)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
