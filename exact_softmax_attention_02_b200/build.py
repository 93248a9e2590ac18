"""Build libfa.so in-tree with nvcc for sm_100a.

    python -m exact_softmax_attention_02_b200.build [--force] [--verbose] [--trace | --debug]

The library is built from csrc/fa_fwd.cu (the fused forward, split-KV,
merge, block-sparse and key-tile variants), csrc/fa_bwd.cu (the backward
pass), csrc/fa_host.cu (the host-buffer forward with pipelined copies) and
csrc/standard_softmax.cu (the comparator's softmax), linked
against the static CUDA runtime; the driver entry point for tensor-map encoding is looked
up at run time, so no libcuda link is needed.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCES = [os.path.join(HERE, "csrc", n)
           for n in ("fa_fwd.cu", "fa_bwd.cu", "fa_host.cu", "standard_softmax.cu")]
DEPENDS = SOURCES + [os.path.join(HERE, "csrc", "sm100.cuh"), os.path.join(HERE, "csrc", "host_util.h"),
                     os.path.join(ROOT, "include", "fa.h")]
OUTPUT = os.path.join(HERE, "libfa.so")
# the same sources built with -DFA_TRACE: SM clock stamps of the forward's
# phases (phase_trace.py reads them); never loaded unless FA_LIBRARY names it
TRACE_OUTPUT = os.path.join(HERE, "libfa_trace.so")
# the same sources built with -DFA_DEBUG: every shared-memory, tensor-memory
# and global index of the forward and merge kernels is checked at run time
# (a failed check raises a status bit and skips the access); loaded only by
# the debug-build tests or when FA_LIBRARY names it
DEBUG_OUTPUT = os.path.join(HERE, "libfa_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I" + os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(output: str = OUTPUT) -> bool:
    if not os.path.exists(output):
        return False
    t = os.path.getmtime(output)
    return all(os.path.getmtime(p) <= t for p in DEPENDS)


def build(force: bool = False, verbose: bool = False, trace: bool = False, debug: bool = False) -> str:
    if trace and debug:
        raise ValueError("build either the trace or the debug library")
    output = TRACE_OUTPUT if trace else DEBUG_OUTPUT if debug else OUTPUT
    if not force and up_to_date(output):
        return output
    tmp = output + ".tmp"
    defs = ["-DFA_TRACE"] if trace else ["-DFA_DEBUG"] if debug else []
    cmd = [nvcc(), *NVCC_FLAGS, *defs, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed: " + " ".join(cmd))
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, output)
    return output


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--trace", action="store_true", help="build libfa_trace.so (-DFA_TRACE) instead")
    ap.add_argument("--debug", action="store_true", help="build libfa_debug.so (-DFA_DEBUG) instead")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, trace=a.trace, debug=a.debug))
