"""Compile the CPU oracle (test infrastructure only) into a shared library.

The oracle is plain C compiled with gcc; it needs no CUDA toolkit.  FMA
contraction and fast-math are disabled so that every double product and sum is
rounded on its own, as the source is written.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "qknorm_oracle.c")
LIBRARY = os.path.join(HERE, "liboracle_qknorm.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(LIBRARY)
            and os.path.getmtime(LIBRARY) >= os.path.getmtime(SOURCE)):
        return LIBRARY
    tmp = LIBRARY + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
           "-Wall", "-Wextra", "-Werror", "-shared", "-fPIC", SOURCE, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force=True))
