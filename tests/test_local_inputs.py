"""The inputs of the exact vs block-sparse experiment: the band layout covers
every (query, key) pair of its window and keeps nothing else, and the local
Q/K carry a positional score of the requested peak."""

import math

import pytest
import torch

from exact_softmax_attention_02_b200.inputs import local_block_layout, make_local_qkv


def _allowed_in_band(i, j, window, causal):
    return (i - window <= j <= i) if causal else abs(i - j) <= window


@pytest.mark.parametrize("N,window,causal,bq,bk,sinks", [
    (300, 40, True, 64, 32, 0), (300, 40, False, 64, 32, 0), (257, 1, True, 32, 64, 1),
    (512, 200, False, 128, 128, 2), (100, 1000, False, 32, 16, 0),
])
def test_band_layout_covers_the_window_and_nothing_more(N, window, causal, bq, bk, sinks):
    lay = local_block_layout(N, window, causal, bq, bk, sinks)
    nqb, nkb = -(-N // bq), -(-N // bk)
    assert len(lay) == nqb and all(len(row) == nkb for row in lay)
    # coverage: every pair inside the band lies in a retained block
    for i in range(N):
        for j in range(N):
            if _allowed_in_band(i, j, window, causal):
                assert lay[i // bq][j // bk], (i, j)
    # no excess: a retained non-sink block holds a key within the widened rows of its block
    for r in range(nqb):
        rows = range(r * bq, min(N, (r + 1) * bq))
        for c in range(nkb):
            if not lay[r][c] or c < sinks:
                continue
            keys = range(c * bk, min(N, (c + 1) * bk))
            lo, hi = rows[0] - window, rows[-1] + (0 if causal else window)
            assert any(lo <= j <= hi for j in keys), (r, c)
    # sinks are kept for every query block
    for r in range(nqb):
        assert all(lay[r][c] for c in range(min(sinks, nkb)))


def test_band_layout_with_a_window_past_n_keeps_everything_non_causal():
    lay = local_block_layout(100, 1000, False, 32, 16)
    assert all(all(row) for row in lay)


def test_local_qkv_shapes_seed_and_shared_features():
    q, k, v = make_local_qkv(2, 3, 50, 16, seed=7)
    assert q.shape == k.shape == v.shape == (2, 3, 50, 16)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    q2, k2, v2 = make_local_qkv(2, 3, 50, 16, seed=7)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    q3, _, _ = make_local_qkv(2, 3, 50, 16, seed=8)
    assert not torch.equal(q, q3)
    # the positional half is the same in Q and K; the content halves differ
    assert torch.equal(q[..., :8], k[..., :8])
    assert not torch.equal(q[..., 8:], k[..., 8:])


@pytest.mark.parametrize("d,peak", [(64, 10.0), (128, 6.0)])
def test_positional_score_at_distance_zero_is_the_peak(d, peak):
    q, k, _ = make_local_qkv(1, 2, 40, d, seed=3, peak=peak)
    pos_q = q[..., : d // 2].double()
    pos_k = k[..., : d // 2].double()
    score = (pos_q * pos_k).sum(-1) / math.sqrt(d)  # same position: a^2 F (cos^2 + sin^2) / sqrt(d)
    # bf16 rounding of each feature: relative error below 2^-8 per factor
    assert torch.allclose(score, torch.full_like(score, peak), rtol=2 ** -6)


def test_head_width_must_be_a_multiple_of_four():
    with pytest.raises(ValueError):
        make_local_qkv(1, 1, 8, 30, seed=0)
