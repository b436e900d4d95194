"""Build step for the CPU oracle (test infrastructure): plain gcc, no CUDA.

The parity oracle (mxfp8_oracle.c) is built ``-O2 -ffp-contract=off`` so
every multiply and add stays a separate IEEE operation.  The timed fp32
baseline (baseline_f32.c) is built ``-O3`` with FMA contraction for
x86-64-v3 (AVX2 + FMA: any current x86 server; not ``-march=native``,
because the built library travels to other hosts).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mxfp8_oracle.c")
BASE = os.path.join(HERE, "baseline_f32.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    srcs = (SRC, BASE, os.path.abspath(__file__))
    if not force and os.path.exists(OUT) and all(os.path.getmtime(OUT) >= os.path.getmtime(f) for f in srcs):
        return OUT
    tmp = OUT + f".tmp{os.getpid()}"
    tmpdir = tempfile.mkdtemp(prefix="oracle_build_")
    o1, o2 = os.path.join(tmpdir, "oracle.o"), os.path.join(tmpdir, "baseline.o")
    common = ["-std=c99", "-fopenmp", "-fPIC", "-Wall", "-Wno-unknown-pragmas"]
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", *common, "-c", SRC, "-o", o1], check=True)
    subprocess.run(["gcc", "-O3", "-march=x86-64-v3", "-ffp-contract=fast", *common, "-c", BASE, "-o", o2],
                   check=True)
    subprocess.run(["gcc", "-shared", "-fopenmp", o1, o2, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, OUT)
    shutil.rmtree(tmpdir, ignore_errors=True)
    return OUT


if __name__ == "__main__":
    print(build(force=True))
