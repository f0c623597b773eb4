"""Compile the plain-C oracle into ``oracle/libgdn_oracle.so`` with gcc.

Test infrastructure: the library built here is loaded only by the tests, the
smoke check and the benchmark's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "gdn_oracle.c")
LIBRARY = os.path.join(HERE, "libgdn_oracle.so")

# -ffp-contract=off keeps every multiply and add a separately rounded double
# operation, so the oracle's rounding follows its source line by line.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Build ``output`` from ``source`` unless it is already newer; return its path."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    cmd = ["gcc", *CFLAGS, "-o", output, source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
