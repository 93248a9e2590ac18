"""The phase-trace summary (host arithmetic only) on a synthetic trace whose
phases have known lengths."""

import numpy as np
import pytest

from exact_softmax_attention_02_b200 import phase_trace as pt


def _synthetic(n_iter=20, period=1000):
    tr = np.zeros((pt.CTAS, pt.ROLES, pt.ITERS, pt.EVENTS), dtype=np.int64)
    for it in range(n_iter):
        base = 10_000 + it * period
        # softmax of tile 0: S seen, loaded +10, max +20, first half +30, done +40
        tr[0, 1, it, :5] = base + np.array([0, 10, 30, 60, 100])
        # MMA issuer: P0 seen 5 after the softmax is done, then 6 phases
        p0 = base + 105
        tr[0, 0, it, :6] = p0 + np.array([0, 50, 150, 200, 260, 380])
    return tr


def test_summary_phase_lengths():
    s = pt.summarize(_synthetic(), cta=0)
    assert s["period"] == pytest.approx(1000)
    assert s["softmax"] == pytest.approx({"load_s": 10, "row_max": 20, "first_half": 30,
                                          "second_half_and_publish": 40, "span": 100})
    assert s["p_published_to_issuer_sees_it"] == pytest.approx(5)
    assert s["p_published_to_next_s_seen"] == pytest.approx(900)
    assert s["mma"] == pytest.approx({"pv0_issue": 50, "s0_issue": 100, "wait_p1": 50, "pv1_issue": 60,
                                      "s1_issue": 120, "to_next_p0": 620})
    # the next S of tile 0 issued at base + 105 + 150; the softmax sees it at base + 1000
    assert s["s0_issued_to_softmax_sees_it"] == pytest.approx(1000 - 255)
    # iterations 4 .. n - 4 count (the head and tail are left out)
    assert s["iterations"] == 20 - 4 - 3


def test_publish_lag_per_warp():
    tr = _synthetic()
    for it in range(20):
        base = 10_000 + it * 1000
        # warps on quarters 1, 2, 3 publish 20, 0 and 40 cycles after quarter 0 (at +100)
        tr[0, 1, it, 5:8] = base + 100 + np.array([20, 0, 40])
    s = pt.summarize(tr, cta=0)
    assert s["publish_lag_tile0"] == pytest.approx([0, 20, 0, 40])
    assert "publish_lag_tile1" not in s


def test_missing_stamps_are_left_out():
    tr = _synthetic()
    tr[0, 1, 8, 3] = 0  # one lost stamp: iteration 8 no longer counts
    s = pt.summarize(tr, cta=0)
    assert s["iterations"] == 20 - 4 - 3 - 1
    assert s["period"] == pytest.approx(1000)


def test_cta_without_stamps_is_an_error():
    with pytest.raises(ValueError):
        pt.summarize(_synthetic(), cta=3)
