"""Compile the scalar C part of the CPU oracle.

Test infrastructure only: the product library never links or loads the
result.  gcc, -O2, -ffp-contract=off (no fused multiply-add), no fast-math,
so every fp32 step is one correctly rounded IEEE operation.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qat_oracle.c")
LIB = os.path.join(HERE, "_liboracle_qat.so")


def build_oracle(force: bool = False) -> str:
    """Build the oracle shared object if missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force=True))
