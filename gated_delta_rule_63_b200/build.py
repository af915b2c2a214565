"""Build libgdr.so (the CUDA library behind include/gdr.h) for sm_100a with nvcc.

    python -m gated_delta_rule_63_b200.build          # writes gated_delta_rule_63_b200/libgdr.so

The library links the CUDA runtime statically and exports only the C ABI.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["gdr_host.cu", "conv.cu", "rmsnorm.cu", "decode.cu", "prefill.cu", "prefill_noalloc.cu", "diag.cu",
           "linear.cu"]
LIB = os.path.join(HERE, "libgdr.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def compile_flags(debug_defines=()):
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                    "-I", os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]
    for d in debug_defines:
        flags += [f"-D{d}"]
    return flags


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def needs_build(out=LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + \
        [os.path.join(ROOT, "include", "gdr.h")]
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(out: str = LIB, defines=(), verbose: bool = False, force: bool = False) -> str:
    """Compile every source and link the shared library; returns its path."""
    if not force and not needs_build(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + compile_flags(defines) + ["-shared", "-o", tmp] + sources()
    if verbose:
        cmd += ["-Xptxas", "-v"]
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
