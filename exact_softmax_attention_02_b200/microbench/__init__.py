"""Microbenchmarks of the forward's MMA issue (standalone CUDA programs).

    python -m exact_softmax_attention_02_b200.microbench [mma_issue | issue_loop | all]

- ``mma_issue.cu``: cycles per tcgen05.mma issued back to back by one thread, in
  the forward's order and TMEM layout, alone and beside TMEM loads and stores,
  ex2 chains, bulk copies into shared memory, barrier polling and barrier waits.
- ``issue_loop.cu``: the forward's MMA issue loop with stand-in producer and
  softmax warps, and what each handshake costs.

Each program prints one JSON line per case and exits non-zero if a bounded
wait gave up. Built with nvcc for sm_100a into ``bin/`` next to this file.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PROGRAMS = ("mma_issue", "issue_loop")


def build(name: str) -> str:
    from ..build import nvcc

    src = os.path.join(HERE, name + ".cu")
    out = os.path.join(HERE, "bin", name)
    deps = [src, os.path.join(HERE, "..", "csrc", "sm100.cuh"), os.path.join(HERE, "..", "csrc", "host_util.h")]
    if os.path.exists(out) and all(os.path.getmtime(p) <= os.path.getmtime(out) for p in deps):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    root = os.path.dirname(os.path.dirname(HERE))
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-I" + os.path.join(root, "include"), "-o", out + ".tmp", src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed: " + " ".join(cmd))
    os.replace(out + ".tmp", out)
    return out


def main(argv=None) -> int:
    which = (argv if argv is not None else sys.argv[1:]) or ["all"]
    names = PROGRAMS if which[0] == "all" else which
    rc = 0
    for name in names:
        if name not in PROGRAMS:
            raise SystemExit(f"unknown microbenchmark {name!r}; one of {PROGRAMS} or all")
        rc |= subprocess.call([build(name)])
    return rc
