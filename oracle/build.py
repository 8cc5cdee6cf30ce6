"""Build the CPU oracle shared library (plain C, gcc, no threads, no BLAS).

Test infrastructure: the oracle is loaded only by the tests, the smoke check
and the bench's CPU-baseline leg.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "twell_oracle.c")
LIB = os.path.join(HERE, "libtwell_oracle.so")


def build(force: bool = False) -> str:
    """Compile ``twell_oracle.c`` into ``libtwell_oracle.so`` when out of date."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    # -ffp-contract=off: keep every multiply and add a separately rounded fp64
    # operation, exactly as written.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fvisibility=hidden", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
