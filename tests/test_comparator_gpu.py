"""GPU parity of the standard (materialising) attention comparator.

The comparator computes the same attention with the N x N scores in memory
(cuBLAS GEMM, this library's row softmax, cuBLAS GEMM).  It is held to the
same tolerances against the float64 oracle as the fused path.
"""

import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import WORKLOADS, make_qkv, sample_rows
from oracle import attention_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run(q, k, v, causal, **kw):
    from exact_softmax_attention_02_b200 import fa
    from exact_softmax_attention_02_b200.comparator import standard_attention

    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = standard_attention(qd, kd, vd, causal=causal, **kw)
    assert fa.device_status_word() == 0
    return o.cpu(), lse.cpu()


def check(o, lse, q, k, v, causal, rows):
    r = rows.numpy()
    d = q.shape[-1]
    ro, rl = attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), 1 / math.sqrt(d),
                            causal, r)
    go = o.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    gl = lse.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    err, lerr = np.abs(go - ro), np.abs(gl - rl)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN and lerr.max() <= LSE_MAX, \
        (err.max(), err.mean(), lerr.max())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(2, 64), (130, 64), (640, 128), (1000, 128)])
def test_standard_every_row(causal, N, d):
    q, k, v = make_qkv(2, 3, N, d, seed=N + d)
    o, lse = run(q, k, v, causal)
    check(o, lse, q, k, v, causal, sample_rows(2, 3, N, 0, 0))


def test_standard_head_groups():
    """A memory budget of one head per group gives the same result."""
    q, k, v = make_qkv(1, 3, 512, 64, seed=4)
    o1, l1 = run(q, k, v, True)
    o2, l2 = run(q, k, v, True, budget_bytes=6 * 512 * 512)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_standard_full_size_sampled():
    w = WORKLOADS["b2h16n8192d128_causal"]
    q, k, v = make_qkv(w.B, w.H, w.N, w.d, w.seed, w.q_std)
    o, lse = run(q, k, v, w.causal)
    check(o, lse, q, k, v, w.causal, sample_rows(w.B, w.H, w.N, 1024, w.seed))
