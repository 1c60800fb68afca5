"""Build liblora_sgmv.so in-tree for sm_100a with nvcc (no JIT, no torch extension)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "liblora_sgmv.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC,-O2", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(HERE, "csrc", "*.h"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in sources() + headers())


def build(force: bool = False, verbose: bool = False, ptxas_v: bool = False, out: str = None,
          defines=()) -> str:
    """Compile every csrc/*.cu into one shared library (default: the in-tree liblora_sgmv.so).
    ``defines`` adds -D flags, e.g. ("LORA_TRACE",) for the phase-traced build written to ``out``."""
    target = out or LIB
    if not force and not defines and out is None and up_to_date():
        return LIB
    tmp = target + ".tmp%d" % os.getpid()
    cmd = [NVCC] + FLAGS + ["-D%s" % d for d in defines] + [
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"), "--threads", "0", "-o", tmp] + sources()
    if ptxas_v:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    trace_out = None
    if "--trace" in sys.argv:
        trace_out = sys.argv[sys.argv.index("--trace") + 1]
    print(build(force="--force" in sys.argv, verbose=True, ptxas_v="--ptxas-v" in sys.argv, out=trace_out,
                defines=("LORA_TRACE",) if trace_out else ()))
