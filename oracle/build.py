"""Compile the CPU oracle (test infrastructure) into oracle/libmx_oracle.so with gcc."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mx_oracle.c")
LIB = os.path.join(HERE, "libmx_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its sources; return its path."""
    deps = [SRC, os.path.join(HERE, "mx_oracle.h")]
    if not force and os.path.exists(LIB) and all(
        os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps
    ):
        return LIB
    # -ffp-contract=off: no fused multiply-adds, every double operation rounds as written.
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-o", LIB + ".tmp", SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
