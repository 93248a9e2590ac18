"""GPU parity of the split-KV forward and of its per-range partial states.

Every key range of a query block leaves a partial state (normalised output
and LSE over that range); the merge combines them.  Both the merged result
and each partial state are compared with the float64 oracle (the partial
ones with the oracle restricted to the same key range).
"""

import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import make_qkv, sample_rows
from oracle import attention_rows, merge_states

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_splitkv(q, k, v, causal, num_splits, keep_workspace=False):
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d = q.shape
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    nbytes = fa.splitkv_workspace_bytes(B, H, N, d, num_splits, causal)
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
    fa.fa_fwd_splitkv(qd, kd, vd, o, lse, workspace=ws, num_splits=num_splits, causal=causal)
    assert fa.device_status_word() == 0
    return o.cpu(), lse.cpu(), ws.cpu()


def check(o, lse, q, k, v, causal, rows):
    d = q.shape[-1]
    r = rows.numpy() if isinstance(rows, torch.Tensor) else rows
    ro, rl = attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), 1 / math.sqrt(d),
                            causal, r)
    go = o.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    gl = lse.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    err, lerr = np.abs(go - ro), np.abs(gl - rl)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN and lerr.max() <= LSE_MAX, \
        (err.max(), err.mean(), lerr.max())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,splits", [(129, 2), (300, 3), (1000, 2), (1000, 8), (2048, 5), (777, 0)])
def test_splitkv_every_row(d, causal, N, splits):
    B, H = 1, 2
    q, k, v = make_qkv(B, H, N, d, seed=N + splits + d)
    o, lse, _ = run_splitkv(q, k, v, causal, splits)
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    check(o, lse, q, k, v, causal, sample_rows(B, H, N, 0, 0))


@pytest.mark.parametrize("causal", [False, True])
def test_partial_states_match_key_range_oracle(causal):
    """Each range's partial (O, LSE) in the workspace is attention over that
    range alone; empty ranges give LSE = -inf and O = 0; the oracle's merge of
    the GPU partials gives the full result."""
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d, splits = 1, 2, 700, 64, 3
    q, k, v = make_qkv(B, H, N, d, seed=5)
    o, lse, ws = run_splitkv(q, k, v, causal, splits)
    n_kv = (N + 127) // 128
    per = (n_kv + splits - 1) // splits
    S = (n_kv + per - 1) // per
    rows_n = B * H * N
    o_part = ws[: S * rows_n * d].reshape(S, B, H, N, d).double().numpy()
    lse_part = ws[S * rows_n * d: S * rows_n * (d + 1)].reshape(S, B, H, N).double().numpy()
    rows = sample_rows(B, H, N, 0, 0).numpy()
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    for s in range(S):
        lo, hi = s * per * 128, min(N, (s + 1) * per * 128)
        ro, rl = attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                1 / math.sqrt(d), causal, rows, key_range=(lo, hi))
        go, gl = o_part[s][b, h, i], lse_part[s][b, h, i]
        empty = np.isneginf(rl)
        assert np.array_equal(np.isneginf(gl), empty)
        assert (go[empty] == 0).all()
        assert np.abs(go[~empty] - ro[~empty]).max() <= 1e-2  # fp32 partial: only P in bf16
        assert np.abs(gl[~empty] - rl[~empty]).max() <= LSE_MAX
    mo, ml = merge_states(o_part[:, b, h, i], lse_part[:, b, h, i])
    assert np.abs(mo - o.double().numpy()[b, h, i]).max() <= 1e-2
    assert np.abs(ml - lse.double().numpy()[b, h, i]).max() <= 1e-4


def test_splitkv_matches_fused_forward():
    from exact_softmax_attention_02_b200 import fa

    q, k, v = make_qkv(2, 3, 1536, 128, seed=9)
    o1, l1, _ = run_splitkv(q, k, v, True, 4)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o2 = torch.empty_like(qd)
    l2 = torch.empty(qd.shape[:3], device="cuda")
    fa.fa_fwd(qd, kd, vd, o2, l2, causal=True)
    assert (o1.float() - o2.cpu().float()).abs().max() <= 1.6e-2
    assert (l1 - l2.cpu()).abs().max() <= 1e-4


def test_splitkv_full_size_small_grid_sampled():
    """A problem with few query blocks (2 heads x 32 blocks), default splits."""
    B, H, N, d = 1, 2, 8192, 128
    q, k, v = make_qkv(B, H, N, d, seed=17)
    o, lse, _ = run_splitkv(q, k, v, True, 0)
    check(o, lse, q, k, v, True, sample_rows(B, H, N, 1024, 17))


def test_one_range_runs_fused_kernel_and_leaves_workspace():
    from exact_softmax_attention_02_b200 import fa

    q, k, v = make_qkv(1, 2, 300, 64, seed=3)
    o, lse, ws = run_splitkv(q, k, v, True, 1)
    assert torch.isnan(ws).all()  # untouched
    check(o, lse, q, k, v, True, sample_rows(1, 2, 300, 0, 0))
