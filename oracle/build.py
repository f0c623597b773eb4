"""Compile the plain-C oracle into ``oracle/libgdn_oracle.so`` with gcc, and
its literal fp32 instantiation of the recurrence into
``oracle/libgdn_oracle_f32.so``.

Test infrastructure: the libraries built here are loaded only by the tests,
the smoke check and the benchmark's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "gdn_oracle.c")
LIBRARY = os.path.join(HERE, "libgdn_oracle.so")
F32_SOURCE = os.path.join(HERE, "gdn_oracle_f32.c")
F32_LIBRARY = os.path.join(HERE, "libgdn_oracle_f32.so")

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


def build_f32(force: bool = False) -> str:
    """Build the fp32 instantiation (the timed CPU baseline); return its path."""
    return build(F32_SOURCE, F32_LIBRARY, force=force)


if __name__ == "__main__":
    force = "--force" in sys.argv
    print(build(force=force))
    print(build_f32(force=force))
