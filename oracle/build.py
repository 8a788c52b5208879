"""Compile the C half of the CPU oracle into ``oracle/liboracle.so``.

Test infrastructure only: the oracle is built so that tests and the bench's
CPU baseline can run it; nothing in the CUDA library links or loads it.
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

HERE = Path(__file__).resolve().parent
SRC = HERE / "qmm_oracle.c"
LIB = HERE / "liboracle.so"

# -ffp-contract=off: no implicit fused multiply-add, so every fp32 step of the
# quantize rule is one correctly rounded IEEE operation.
CFLAGS = ["-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> Path:
    """Build liboracle.so if missing or older than its source; return its path."""
    if not force and LIB.exists() and LIB.stat().st_mtime >= SRC.stat().st_mtime:
        return LIB
    tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
    cmd = ["gcc", *CFLAGS, str(SRC), "-o", str(tmp), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
