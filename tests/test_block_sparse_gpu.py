"""GPU parity of the block-sparse forward (fa_fwd_block_sparse).

The kernel is the fused forward visiting only the key tiles each 256-row
query block retains.  It is compared with the float64 oracle's block-sparse
definition (the softmax over retained blocks), and, with every block
retained, with fa_fwd bit for bit.  Malformed lists are masked on the device
and reported as FA_ERR_LAYOUT.
"""

import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import local_block_layout, make_local_qkv, make_qkv, sample_rows
from oracle import block_sparse_attention_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
BQ, BK = 256, 128


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def run_sparse(q, k, v, layout, causal):
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d = q.shape
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    rp, ci = fa.block_layout_to_csr(layout, device="cuda")
    fa.fa_fwd_block_sparse(qd, kd, vd, o, rp, ci, lse, causal=causal)
    assert fa.device_status_word() == 0
    return o.cpu(), lse.cpu()


def check(o, lse, q, k, v, causal, rows, layout):
    d = q.shape[-1]
    r = rows.numpy() if isinstance(rows, torch.Tensor) else rows
    ro, rl = block_sparse_attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                         1 / math.sqrt(d), causal, r, np.asarray(layout, bool), BQ, BK)
    go = o.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    gl = lse.double().numpy()[r[:, 0], r[:, 1], r[:, 2]]
    empty = np.isneginf(rl)
    assert (go[empty] == 0).all() and np.isneginf(gl[empty]).all()
    err, lerr = np.abs(go - ro), np.abs(gl[~empty] - rl[~empty])
    assert err.max() <= O_MAX and err.mean() <= O_MEAN, (err.max(), err.mean())
    if lerr.size:
        assert lerr.max() <= LSE_MAX, lerr.max()


def random_layout(N, seed, density=0.5):
    rng = np.random.default_rng(seed)
    lay = rng.random((-(-N // BQ), -(-N // BK))) < density
    lay[0, :] = False  # a query block with no retained key
    return lay


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 1000, 1536])
def test_random_layouts_every_row(d, causal, N):
    B, H = 2, 2
    q, k, v = make_qkv(B, H, N, d, seed=N + d + causal)
    lay = random_layout(N, N + d)
    o, lse = run_sparse(q, k, v, lay, causal)
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    check(o, lse, q, k, v, causal, sample_rows(B, H, N, 0, 0), lay)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 200, 777, 2048])
def test_full_layout_equals_fa_fwd_bit_for_bit(d, causal, N):
    from exact_softmax_attention_02_b200 import fa

    B, H = 1, 3
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=N * 3 + d))
    lay = np.ones((-(-N // BQ), -(-N // BK)), bool)
    o_s, l_s = run_sparse(q, k, v, lay, causal)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device="cuda")
    fa.fa_fwd(q, k, v, o, lse, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o_s, o.cpu()) and torch.equal(l_s, lse.cpu())


@pytest.mark.parametrize("causal", [False, True])
def test_band_layout_on_local_inputs_large(causal):
    """A band of key blocks (plus one sink block) at N = 8192, d = 128, sampled rows."""
    B, H, N, d = 1, 4, 8192, 128
    q, k, v = make_local_qkv(B, H, N, d, seed=11)
    lay = local_block_layout(N, 512, causal, BQ, BK, sinks=1)
    o, lse = run_sparse(q, k, v, lay, causal)
    check(o, lse, q, k, v, causal, sample_rows(B, H, N, 1024, 11), lay)


def test_causal_blocks_above_the_diagonal_are_skipped():
    """Only blocks above the diagonal retained: causal rows of a block that sees none of
    them get O = 0 and LSE = -inf; rows that see part of a diagonal block are exact."""
    B, H, N, d = 1, 1, 1024, 64
    q, k, v = make_qkv(B, H, N, d, seed=3)
    lay = np.zeros((4, 8), bool)
    lay[0, 1] = True   # keys 128..255 for rows 0..255: rows < 128 see nothing
    lay[1, 7] = True   # keys past every row of block 1: all empty
    lay[2, 4] = True   # keys 512..639: rows 512..767 see part of it
    o, lse = run_sparse(q, k, v, lay, True)
    check(o, lse, q, k, v, True, sample_rows(B, H, N, 0, 0), lay)
    assert np.isneginf(lse[0, 0, :128].numpy()).all() and (o[0, 0, :128] == 0).all()
    assert np.isneginf(lse[0, 0, 256:512].numpy()).all()


def test_malformed_lists_are_masked_and_reported():
    """Out-of-range and out-of-order entries raise FA_ERR_LAYOUT; nothing faults."""
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d = 1, 1, 512, 64
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=9))
    o = torch.empty_like(q)
    for rp, ci in (([0, 2, 3], [0, 9, 1]),      # 9 >= 4 key blocks
                   ([0, 2, 4], [1, 0, 2, 3]),   # descending inside block 0
                   ([0, 3, 2], [0, 1, 2]),      # row_ptr decreasing
                   ([0, 1, 5], [0, 1, 2, 3])):  # row_ptr past nnz
        rpt = torch.tensor(rp, dtype=torch.int32, device="cuda")
        cit = torch.tensor(ci, dtype=torch.int32, device="cuda")
        fa.fa_fwd_block_sparse(q, k, v, o, rpt, cit)
        assert fa.device_status(None) == fa.FA_ERR_LAYOUT
    # a good list afterwards reports nothing
    rpt = torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda")
    cit = torch.tensor([0, 3], dtype=torch.int32, device="cuda")
    fa.fa_fwd_block_sparse(q, k, v, o, rpt, cit)
    assert fa.device_status(None) == fa.FA_OK
