"""GPU parity of the forward in every tile shape of the sweep (fa_fwd_tile_config).

The tile-size sweep runs the fused kernel with 64-key tiles as well as the
default 128, and with one 128-row query tile per CTA as well as the default
two.  Every shape must compute the same attention: every row is checked
against the float64 oracle on small and ragged problems, sampled rows on a
large one, and the shapes against the default.
"""

import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
from oracle import attention_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


SHAPES = [(256, 64), (128, 128), (128, 64)]  # (query rows per CTA, keys per tile)


def run(q, k, v, causal, key_tile, query_rows=256):
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d = q.shape
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    fa.fa_fwd_tile_config(qd, kd, vd, o, lse, query_rows=query_rows, key_tile=key_tile, causal=causal)
    assert fa.device_status_word() == 0
    return o.cpu(), lse.cpu()


def check(o, lse, q, k, v, causal, rows):
    d = q.shape[-1]
    r = rows.numpy()
    ro, rl = attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), 1 / math.sqrt(d),
                            causal, r)
    go = o.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    gl = lse.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    err, lerr = np.abs(go - ro), np.abs(gl - rl)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN and lerr.max() <= LSE_MAX, \
        (err.max(), err.mean(), lerr.max())


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 63, 64, 65, 200, 1000, 1536])
def test_tile_shapes_every_row(shape, d, causal, N):
    B, H = 1, 2
    q, k, v = make_qkv(B, H, N, d, seed=7 * N + d)
    o, lse = run(q, k, v, causal, shape[1], shape[0])
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    check(o, lse, q, k, v, causal, sample_rows(B, H, N, 0, 0))


@pytest.mark.parametrize("shape", SHAPES)
def test_tile_shapes_large_sampled_and_close_to_default(shape):
    w = WORKLOADS["b2h16n8192d128_causal"]
    q, k, v = make_workload_inputs(w)
    o_s, l_s = run(q, k, v, w.causal, shape[1], shape[0])
    check(o_s, l_s, q, k, v, w.causal, sample_rows(w.B, w.H, w.N, 2048, w.seed))
    o_d, l_d = run(q, k, v, w.causal, 128, 256)
    # same attention, different tile boundaries: rounding-level differences only
    assert (o_s.float() - o_d.float()).abs().max().item() <= 2e-2
    assert (l_s - l_d).abs().max().item() <= 1e-3


def test_one_query_tile_per_cta_equals_default_bit_for_bit():
    """With 128 keys per tile, one query tile per CTA runs the same per-row
    arithmetic as the default, so the results are identical."""
    q, k, v = make_qkv(2, 3, 1000, 128, seed=77)
    for causal in (False, True):
        o1, l1 = run(q, k, v, causal, 128, 128)
        o2, l2 = run(q, k, v, causal, 128, 256)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
