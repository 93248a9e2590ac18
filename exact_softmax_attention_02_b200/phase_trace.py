"""Phase trace of the fused forward: where one iteration's cycles go.

    python -m exact_softmax_attention_02_b200.phase_trace [--workload NAME] [--out trace.npy]
    python -m exact_softmax_attention_02_b200.phase_trace --from trace.npy

The first form builds ``libfa_trace.so`` (the library compiled with
``-DFA_TRACE``), runs one ``fa_fwd`` launch of the workload on ``cuda:0`` with a
trace buffer attached, saves the raw stamps and prints the summary.  The
second form summarises a saved trace on any host.

The trace build stamps the SM clock (``clock64``) at fixed points of the first
``CTAS`` CTAs, for the first ``ITERS`` key tiles each, into
``[CTAS][4 roles][ITERS][8 events]`` 64-bit slots (zero where nothing was
stamped).  Roles and events, per iteration ``it``:

- role 0, the MMA issuer: ``3t`` P of query tile t seen, ``3t + 1`` the PV
  products of tile t issued, ``3t + 2`` the next S product of tile t issued and
  committed (t = 0, 1);
- roles 1 and 2, the softmax warpgroup of tile 0 and of tile 1: lane 0 of the
  warp on TMEM lane quarter 0 stamps 0 S seen in TMEM, 1 S loaded into
  registers, 2 row maximum taken, 3 first half of P stored, 4 the tile done
  (P published, denominator updated); lane 0 of the warps on quarters 1, 2, 3
  stamps 5, 6, 7 when its warp has published P;
- role 3, the MMA issuer again: 0 the V tile of the iteration landed, 1 the
  next K tile landed.

The summary averages over iterations whose stamps are all present, leaving out
the first and last few, where the pipeline fills and drains.
"""

from __future__ import annotations

import argparse
import ctypes
import json
import os
import sys

import numpy as np

CTAS = 16
ITERS = 64
ROLES = 4
EVENTS = 8


def summarize(trace: np.ndarray, cta: int = 0, skip_head: int = 4, skip_tail: int = 3) -> dict:
    """Mean cycles of each phase for one CTA of a ``[CTAS, 4, ITERS, 8]`` trace.

    An iteration ``it`` counts when the MMA stamps of ``it`` and ``it + 1`` and
    the tile-0 softmax stamps of ``it`` and ``it + 1`` are all present."""
    t = np.asarray(trace, dtype=np.int64).reshape(-1, ROLES, ITERS, EVENTS)[cta]
    mma, sm0 = t[0], t[1]
    n = int((mma[:, 0] > 0).sum())
    its = [i for i in range(skip_head, n - skip_tail)
           if i + 1 < ITERS and (mma[i, :6] > 0).all() and mma[i + 1, 0] > 0
           and (sm0[i, :5] > 0).all() and sm0[i + 1, 0] > 0]
    if not its:
        raise ValueError(f"no complete iterations in CTA {cta} (MMA stamps in {n} iterations)")

    def mean(f):
        return float(np.mean([f(i) for i in its]))

    return {
        "cta": cta,
        "iterations": len(its),
        "period": mean(lambda i: mma[i + 1, 0] - mma[i, 0]),
        "softmax": {
            "load_s": mean(lambda i: sm0[i, 1] - sm0[i, 0]),
            "row_max": mean(lambda i: sm0[i, 2] - sm0[i, 1]),
            "first_half": mean(lambda i: sm0[i, 3] - sm0[i, 2]),
            "second_half_and_publish": mean(lambda i: sm0[i, 4] - sm0[i, 3]),
            "span": mean(lambda i: sm0[i, 4] - sm0[i, 0]),
        },
        "p_published_to_next_s_seen": mean(lambda i: sm0[i + 1, 0] - sm0[i, 4]),
        "p_published_to_issuer_sees_it": mean(lambda i: mma[i, 0] - sm0[i, 4]),
        "mma": {
            "pv0_issue": mean(lambda i: mma[i, 1] - mma[i, 0]),
            "s0_issue": mean(lambda i: mma[i, 2] - mma[i, 1]),
            "wait_p1": mean(lambda i: mma[i, 3] - mma[i, 2]),
            "pv1_issue": mean(lambda i: mma[i, 4] - mma[i, 3]),
            "s1_issue": mean(lambda i: mma[i, 5] - mma[i, 4]),
            "to_next_p0": mean(lambda i: mma[i + 1, 0] - mma[i, 5]),
        },
        "s0_issued_to_softmax_sees_it": mean(lambda i: sm0[i + 1, 0] - mma[i, 2]),
        **publish_lag(t, its),
    }


def publish_lag(t: np.ndarray, its) -> dict:
    """How long after the first warp of a softmax warpgroup each of its four
    warps published P (mean cycles over the iterations where all four stamped),
    per query tile; empty when the trace has no per-warp stamps."""
    out = {}
    for tile in (0, 1):
        pubs = t[1 + tile, :, 4:8]
        rows = [i for i in its if (pubs[i] > 0).all()]
        if rows:
            p = pubs[rows].astype(np.float64)
            lag = (p - p.min(axis=1, keepdims=True)).mean(axis=0)
            out[f"publish_lag_tile{tile}"] = [float(x) for x in lag]
    return out


def record(workload: str, out: str | None) -> np.ndarray:
    """One traced launch of ``workload`` on cuda:0; returns the raw stamps."""
    from . import build

    os.environ["FA_LIBRARY"] = build.build(trace=True)
    import torch

    from . import fa
    from .inputs import WORKLOADS, make_qkv

    if not torch.cuda.is_available():
        raise SystemExit("the trace needs a CUDA device")
    w = WORKLOADS[workload]
    q, k, v = (x.to("cuda:0") for x in make_qkv(w.B, w.H, w.N, w.d, w.seed, w.q_std))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    lib = fa._load()
    lib.fa_trace_set.argtypes = [ctypes.c_void_p]
    lib.fa_trace_set.restype = ctypes.c_int
    buf = torch.zeros(CTAS * ROLES * ITERS * EVENTS, dtype=torch.int64, device=q.device)
    fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)  # warm-up, untraced
    torch.cuda.synchronize()
    if lib.fa_trace_set(ctypes.c_void_p(buf.data_ptr())) != 0:
        raise RuntimeError("fa_trace_set failed")
    try:
        fa.fa_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)
        torch.cuda.synchronize()
    finally:
        lib.fa_trace_set(None)
    if fa.device_status() != 0:
        raise RuntimeError("the traced launch reported a device failure")
    trace = buf.cpu().numpy().reshape(CTAS, ROLES, ITERS, EVENTS)
    if out:
        np.save(out, trace)
    return trace


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", default="b2h16n8192d128_causal")
    ap.add_argument("--out", default=None, help="save the raw stamps (.npy)")
    ap.add_argument("--from", dest="src", default=None, help="summarise a saved trace instead of recording")
    ap.add_argument("--ctas", type=int, default=2, help="CTAs to summarise")
    a = ap.parse_args(argv)
    trace = np.load(a.src) if a.src else record(a.workload, a.out)
    for c in range(a.ctas):
        print(json.dumps(summarize(trace, c)))
    return 0


if __name__ == "__main__":
    sys.exit(main())
