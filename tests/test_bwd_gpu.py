"""GPU parity of the backward pass (dQ, dK, dV) against the float64 oracle.

The forward runs through fa_fwd (its bf16 O and fp32 LSE feed the backward,
as in training); the oracle differentiates the exact definition from the
same bf16 inputs.  Tolerance, relative to the largest reference magnitude of
each gradient: P and dS enter the tensor-core products rounded to bf16
(relative 2^-9 each), O is bf16, and the outputs are rounded to bf16, so a
few units of 2^-9 per element are expected; the test allows max error
2^-5 and mean error 2^-9 of max|reference|.  A gradient that vanishes exactly
(dQ and dK with a single key) is measured against 2^-4 of the largest
magnitude among the three gradients instead.
"""

import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import make_qkv
from oracle import attention_backward

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 2.0 ** -5, 2.0 ** -9


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_bwd(q, k, v, do, causal):
    from exact_softmax_attention_02_b200 import fa

    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:3], device="cuda")
    fa.fa_fwd(qd, kd, vd, o, lse, causal=causal)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    fa.fa_bwd(qd, kd, vd, o, dod, lse, dq, dk, dv, causal=causal)
    assert fa.device_status_word() == 0
    return dq.cpu(), dk.cpu(), dv.cpu()


def compare(name, got, ref, report, floor=0.0):
    g = got.double().numpy()
    scale = max(np.abs(ref).max(), floor, 1e-30)
    err = np.abs(g - ref)
    report.append((name, err.max() / scale, err.mean() / scale))
    assert np.isfinite(g).all(), name
    assert err.max() <= MAX_REL * scale, (name, err.max() / scale)
    assert err.mean() <= MEAN_REL * scale, (name, err.mean() / scale)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 200, 256, 300, 640])
def test_backward_every_element(d, causal, N):
    B, H = 1, 2
    q, k, v = make_qkv(B, H, N, d, seed=N + 3 * d + int(causal))
    do = make_qkv(B, H, N, d, seed=10_000 + N)[0]
    dq, dk, dv = run_bwd(q, k, v, do, causal)
    rq, rk, rv, _ = attention_backward(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                       do.float().numpy(), 1 / math.sqrt(d), causal)
    report = []
    floor = 2.0 ** -4 * max(np.abs(r).max() for r in (rq, rk, rv))
    compare("dq", dq, rq, report, floor)
    compare("dk", dk, rk, report, floor)
    compare("dv", dv, rv, report, floor)
    print(report)


def test_backward_peaked_rows():
    """Q ~ N(0, 4^2): sharply peaked attention."""
    q, k, v = make_qkv(1, 2, 512, 128, seed=7, q_std=4.0)
    do = make_qkv(1, 2, 512, 128, seed=8)[0]
    dq, dk, dv = run_bwd(q, k, v, do, True)
    rq, rk, rv, _ = attention_backward(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                       do.float().numpy(), 1 / math.sqrt(128), True)
    report = []
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        compare(name, g, r, report)


def test_backward_full_size_two_heads():
    """B=2, H=16, N=8192, d=128 causal: every element of the first and last head."""
    B, H, N, d = 2, 16, 8192, 128
    q, k, v = make_qkv(B, H, N, d, seed=2)
    do = make_qkv(B, H, N, d, seed=12)[0]
    dq, dk, dv = run_bwd(q, k, v, do, True)
    for b, h in ((0, 0), (B - 1, H - 1)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv, _ = attention_backward(q[sl].float().numpy(), k[sl].float().numpy(),
                                           v[sl].float().numpy(), do[sl].float().numpy(),
                                           1 / math.sqrt(d), True)
        report = []
        compare("dq", dq[sl], rq, report)
        compare("dk", dk[sl], rk, report)
        compare("dv", dv[sl], rv, report)
