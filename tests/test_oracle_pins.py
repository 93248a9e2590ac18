"""Pins of the float64 oracle to facts the pages and mathematics fix.

Each test ties an oracle function to something other than itself: a value a
page prints, a closed form, an invariant the pages state, or brute force.
The mutation tests at the end plant plausible mistakes in copies of the
oracle (on the CPU) and check that the pin set rejects every one.
"""

import math

import numpy as np
import pytest

from conftest import floats, load_golden
from oracle import (
    attention_full,
    attention_rows,
    brute_force_attention,
    flops_for_rows,
    merge_block,
    online_attention_rows,
    scalar_online_weighted_sum,
    scalar_softmax_weighted_sum,
)


def scalar_problem(scores, values, n_queries=None):
    """Embed scalar scores/values as a d=1 attention head with q = 1, scale = 1."""
    n = len(scores)
    nq = n if n_queries is None else n_queries
    q = np.ones((1, 1, nq, 1))
    k = np.asarray(scores, dtype=np.float64).reshape(1, 1, n, 1)
    v = np.asarray(values, dtype=np.float64).reshape(1, 1, n, 1)
    return q, k, v


def all_rows(B, H, N):
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], 1)


# ---------------------------------------------------------------------------
# Worked examples printed or asserted on the pages
# ---------------------------------------------------------------------------

def test_three_scores_printed_value():
    g = load_golden("three_scores.txt")
    scores, values = floats(g["scores"]), floats(g["values"])
    printed = float(g["printed_output"])
    q, k, v = scalar_problem(scores, values)
    o, lse = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, 3))
    for r in range(3):
        assert round(o[r, 0], int(g["printed_decimals"])) == printed
    # closed form of the same sum: (10 + 20e + 30e^2) / (1 + e + e^2)
    e = math.e
    closed = (10 + 20 * e + 30 * e * e) / (1 + e + e * e)
    assert math.isclose(o[0, 0], closed, rel_tol=1e-14)
    # LSE = ln(1 + e + e^2) = 2 + ln(1 + e^-1 + e^-2)
    assert math.isclose(lse[0], math.log(1 + e + e * e), rel_tol=1e-14)
    assert math.isclose(lse[0], 2.4076059644443806, rel_tol=1e-14)


def test_three_scores_shift_by_1000():
    g = load_golden("three_scores.txt")
    scores, values = floats(g["scores"]), floats(g["values"])
    shift = float(g["shift"])
    tol = float(g["rel_tol"])
    q, k, v = scalar_problem(scores, values)
    base, base_lse = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, 3))
    q2, k2, v2 = scalar_problem([s + shift for s in scores], values)
    shifted, shifted_lse = attention_rows(q2, k2, v2, 1.0, False, all_rows(1, 1, 3))
    assert np.allclose(shifted, base, rtol=tol, atol=0)
    # the log-sum-exp moves by exactly the shift
    assert np.allclose(shifted_lse - shift, base_lse, rtol=0, atol=1e-12)
    # the online path agrees at the page's tolerance
    on, _ = online_attention_rows(q2, k2, v2, 1.0, False, all_rows(1, 1, 3), tile=1)
    assert np.allclose(on, base, rtol=tol, atol=0)


def test_four_scores_blocks_of_two():
    g = load_golden("four_scores_blocks.txt")
    scores, values = floats(g["scores"]), floats(g["values"])
    block, tol = int(g["block"]), float(g["abs_tol"])
    e = math.e
    # e^(1-1002) and e^(2-1002) underflow to 0 in float64, so the exact
    # float64 result is the two-key closed form (4 e^-1 + 8) / (e^-1 + 1).
    closed = (4 + 8 * e) / (1 + e)
    closed_lse = 1002 + math.log(1 + math.exp(-1))
    q, k, v = scalar_problem(scores, values)
    rows = all_rows(1, 1, 4)
    full, full_lse = attention_rows(q, k, v, 1.0, False, rows)
    tiled, tiled_lse = online_attention_rows(q, k, v, 1.0, False, rows, tile=block)
    assert abs(full[0, 0] - closed) < tol
    assert abs(tiled[0, 0] - closed) < tol
    assert abs(full_lse[0] - closed_lse) < 1e-12
    assert abs(tiled_lse[0] - closed_lse) < 1e-12
    # the scalar running-statistics form of the same example
    so, sl = scalar_online_weighted_sum(scores, values, block=block)
    assert abs(so - closed) < tol and abs(sl - closed_lse) < 1e-12


def test_lse_blocks_running_max_and_sum():
    g = load_golden("lse_blocks.txt")
    blocks = [floats(b) for b in g["block"]]
    flat = [x for b in blocks for x in b]
    exact_lse = math.log(math.fsum(math.exp(x) for x in flat))
    # running statistics over the three blocks, via the oracle's merge
    m, total, acc = np.array([-np.inf]), np.zeros(1), np.zeros((1, 1))
    for b in blocks:
        m, total, acc = merge_block(m, total, acc, np.array([b]), np.ones((len(b), 1)))
    assert m[0] == float(g["running_max"])
    assert math.isclose(total[0], math.fsum(math.exp(x - 4.1) for x in flat), rel_tol=1e-14)
    assert math.isclose(m[0] + math.log(total[0]), exact_lse, rel_tol=1e-14)
    # and the full-row LSE of the six scores
    q, k, v = scalar_problem(flat, [0.0] * 6)
    _, lse = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, 6))
    assert math.isclose(lse[0], exact_lse, rel_tol=1e-14)


def test_rescale_both_numerator_and_denominator():
    g = load_golden("rescale_5_to_10.txt")
    old_max, new_max = float(g["old_max"]), float(g["new_max"])
    factor = math.exp(float(g["factor_exponent"]))
    s1, v1 = [old_max, 3.0], [1.0, 2.0]
    s2, v2 = [new_max, 7.0], [3.0, 4.0]
    m, total, acc = merge_block(np.array([-np.inf]), np.zeros(1), np.zeros((1, 1)),
                                np.array([s1]), np.array(v1).reshape(2, 1))
    assert m[0] == old_max
    l_old, u_old = total[0], acc[0, 0]
    m, total, acc = merge_block(m, total, acc, np.array([s2]), np.array(v2).reshape(2, 1))
    assert m[0] == new_max
    new_l = 1 + math.exp(7 - 10)
    new_u = 3 + 4 * math.exp(7 - 10)
    assert math.isclose(total[0], l_old * factor + new_l, rel_tol=1e-15)
    assert math.isclose(acc[0, 0], u_old * factor + new_u, rel_tol=1e-15)
    full, _ = scalar_softmax_weighted_sum(s1 + s2, v1 + v2)
    assert math.isclose(acc[0, 0] / total[0], full, rel_tol=1e-14)
    # rescaling only one of the two changes the result
    assert not math.isclose((u_old + new_u) / (l_old * factor + new_l), full, rel_tol=1e-3)
    assert not math.isclose((u_old * factor + new_u) / (l_old + new_l), full, rel_tol=1e-3)


def test_block_average_is_not_softmax():
    """Averaging per-block softmax results is not the global softmax."""
    g = load_golden("three_scores.txt")
    scores, values = floats(g["scores"]), floats(g["values"])
    first, _ = scalar_softmax_weighted_sum(scores[:2], values[:2])
    second, _ = scalar_softmax_weighted_sum(scores[2:], values[2:])
    averaged = 0.5 * (first + second)
    q, k, v = scalar_problem(scores, values)
    o, _ = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, 3))
    assert abs(averaged - o[0, 0]) > 1.0
    assert round(o[0, 0], 6) == float(g["printed_output"])


def test_causal_rows_of_three_scores():
    q, k, v = scalar_problem([0.0, 1.0, 2.0], [10.0, 20.0, 30.0])
    o, lse = attention_rows(q, k, v, 1.0, True, all_rows(1, 1, 3))
    e = math.e
    assert o[0, 0] == 10.0 and lse[0] == 0.0  # one allowed key: its value, its score
    assert math.isclose(o[1, 0], (10 + 20 * e) / (1 + e), rel_tol=1e-14)
    assert math.isclose(lse[1], math.log(1 + e), rel_tol=1e-14)
    assert math.isclose(o[2, 0], (10 + 20 * e + 30 * e * e) / (1 + e + e * e), rel_tol=1e-14)


def test_random_scalar_rows_online_equals_full():
    """390 random scalar rows of lengths 1..39, as the page checked (own seed)."""
    rng = np.random.default_rng(20221027)
    for case in range(390):
        n = 1 + case % 39
        scores = (rng.standard_normal(n) * 5).tolist()
        values = rng.standard_normal(n).tolist()
        ref, ref_lse = scalar_softmax_weighted_sum(scores, values)
        on, on_lse = scalar_online_weighted_sum(scores, values, block=1)
        assert math.isclose(on, ref, rel_tol=1e-12, abs_tol=1e-12)
        assert math.isclose(on_lse, ref_lse, rel_tol=1e-12)
        q, k, v = scalar_problem(scores, values, n_queries=1)
        o, lse = attention_rows(q, k, v, 1.0, False, np.array([[0, 0, 0]]))
        assert math.isclose(o[0, 0], ref, rel_tol=1e-12, abs_tol=1e-12)
        assert math.isclose(lse[0], ref_lse, rel_tol=1e-12)


# ---------------------------------------------------------------------------
# Closed forms and brute force on small attention heads
# ---------------------------------------------------------------------------

def test_constant_values_and_equal_keys():
    rng = np.random.default_rng(7)
    B, H, N, d = 1, 2, 9, 4
    q = rng.standard_normal((B, H, N, d))
    k = np.broadcast_to(rng.standard_normal((1, 1, 1, d)), (B, H, N, d)).copy()
    v = rng.standard_normal((B, H, N, d))
    for causal in (False, True):
        o, lse = attention_full(q, k, v, 0.5, causal)
        for i in range(N):
            n_allowed = i + 1 if causal else N
            mean_v = v[:, :, :n_allowed, :].mean(axis=2)
            assert np.allclose(o[:, :, i, :], mean_v, rtol=1e-13, atol=1e-14)
            s = 0.5 * (q[:, :, i, :] * k[:, :, 0, :]).sum(-1)
            assert np.allclose(lse[:, :, i], s + math.log(n_allowed), rtol=1e-13)
    # every value row equal: the output is that row, whatever the scores
    vc = np.broadcast_to(rng.standard_normal((1, 1, 1, d)), (B, H, N, d)).copy()
    kr = rng.standard_normal((B, H, N, d)) * 3
    o, _ = attention_full(q, kr, vc, 1.0, False)
    assert np.allclose(o, vc, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    N, d = int(rng.integers(1, 18)), int(rng.integers(1, 9))
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, N, d)) * 1.5
    v = rng.standard_normal((B, H, N, d))
    scale = float(rng.uniform(0.2, 1.2))
    causal = bool(seed % 2)
    bo, bl = brute_force_attention(q, k, v, scale, causal)
    bo, bl = np.array(bo), np.array(bl)
    o, lse = attention_full(q, k, v, scale, causal)
    assert np.allclose(o, bo, rtol=1e-12, atol=1e-13)
    assert np.allclose(lse, bl, rtol=1e-12, atol=1e-13)
    on, onl = online_attention_rows(q, k, v, scale, causal, all_rows(B, H, N), tile=3)
    assert np.allclose(on.reshape(o.shape), bo, rtol=1e-12, atol=1e-13)
    assert np.allclose(onl.reshape(lse.shape), bl, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_online_matches_full_multi_tile(causal):
    """Independent paths agree over several 64-key tiles and a ragged tail."""
    rng = np.random.default_rng(5)
    B, H, N, d = 2, 2, 200, 16
    q = rng.standard_normal((B, H, N, d)) * 3
    k = rng.standard_normal((B, H, N, d))
    v = rng.standard_normal((B, H, N, d))
    rows = all_rows(B, H, N)
    o, l = attention_rows(q, k, v, 0.25, causal, rows)
    on, onl = online_attention_rows(q, k, v, 0.25, causal, rows)
    assert np.allclose(on, o, rtol=1e-12, atol=1e-13)
    assert np.allclose(onl, l, rtol=1e-12, atol=1e-13)


def test_row_subset_and_order_do_not_matter():
    rng = np.random.default_rng(9)
    q, k, v = (rng.standard_normal((2, 3, 20, 8)) for _ in range(3))
    rows = all_rows(2, 3, 20)
    o, l = attention_rows(q, k, v, 0.3, True, rows)
    perm = rng.permutation(len(rows))[:17]
    o2, l2 = attention_rows(q, k, v, 0.3, True, rows[perm])
    assert np.array_equal(o2, o[perm]) and np.array_equal(l2, l[perm])


def test_large_magnitude_rows_stay_finite():
    """Scores far beyond exp's range: max subtraction keeps everything finite."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 1, 64, 8)) * 200
    k = rng.standard_normal((1, 1, 64, 8)) * 200
    v = rng.standard_normal((1, 1, 64, 8))
    o, l = attention_full(q, k, v, 1.0, True)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l))
    # peaked rows: output equals the value of the best key
    s = (q[0, 0] @ k[0, 0].T)
    s = np.where(np.tril(np.ones((64, 64), bool)), s, -np.inf)
    best = s.argmax(1)
    gap = np.sort(s, 1)[:, -1] - np.sort(s, 1)[:, -2]
    sharp = gap > 50
    assert sharp.sum() > 10
    assert np.allclose(o[0, 0][sharp], v[0, 0][best[sharp]], atol=1e-12)


def test_flop_count_convention():
    g = load_golden("score_counts.txt")
    n = int(g["tokens"])
    assert n * n == int(g["pairwise_scores"])
    assert int(g["tile_rows"]) * int(g["tile_cols"]) == int(g["tile_scores"])
    d = 64
    rows = all_rows(1, 1, n)
    # 2 N^2 d multiply-adds per head = 4 N^2 d FLOPs
    assert flops_for_rows(rows, n, d, False) == 4.0 * n * n * d
    assert flops_for_rows(rows, n, d, True) == 4.0 * d * n * (n + 1) / 2
    nb = int(g["score_matrix_tokens"])
    assert nb * nb * int(g["score_matrix_bytes_per_element"]) == int(g["score_matrix_mib"]) << 20


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle must fail at least one pin
# ---------------------------------------------------------------------------

def _pin_failures(impl):
    """Run a compact copy of the pins above against ``impl`` (same signature
    as attention_rows); return the names of the pins it fails."""
    fails = []
    e = math.e
    q, k, v = scalar_problem([0.0, 1.0, 2.0], [10.0, 20.0, 30.0])
    o, l = impl(q, k, v, 1.0, False, all_rows(1, 1, 3))
    if round(o[0, 0], 6) != 25.752104:
        fails.append("three_scores")
    if not math.isclose(l[0], 2.4076059644443806, rel_tol=1e-12):
        fails.append("three_scores_lse")
    q, k, v = scalar_problem([1.0, 2.0, 1001.0, 1002.0], [2.0, -1.0, 4.0, 8.0])
    o, l = impl(q, k, v, 1.0, False, all_rows(1, 1, 4))
    if not (np.isfinite(o[0, 0]) and abs(o[0, 0] - (4 + 8 * e) / (1 + e)) < 1e-12):
        fails.append("four_scores")
    q, k, v = scalar_problem([0.0, 1.0, 2.0], [10.0, 20.0, 30.0])
    o, l = impl(q, k, v, 1.0, True, all_rows(1, 1, 3))
    if not (o[0, 0] == 10.0 and math.isclose(o[1, 0], (10 + 20 * e) / (1 + e), rel_tol=1e-12)):
        fails.append("causal_rows")
    rng = np.random.default_rng(42)
    B, H, N, d = 2, 2, 7, 3
    qq = rng.standard_normal((B, H, N, d))
    kk = rng.standard_normal((B, H, N, d))
    vv = rng.standard_normal((B, H, N, d))
    for causal in (False, True):
        bo, bl = brute_force_attention(qq, kk, vv, 0.7, causal)
        o, l = impl(qq, kk, vv, 0.7, causal, all_rows(B, H, N))
        if not (np.allclose(o, np.array(bo).reshape(-1, d), rtol=1e-12, atol=1e-13)
                and np.allclose(l, np.array(bl).ravel(), rtol=1e-12, atol=1e-13)):
            fails.append(f"brute_force_causal{int(causal)}")
    return fails


def _mutant(kind):
    def impl(q, k, v, scale, causal, rows):
        rows = np.asarray(rows).reshape(-1, 3)
        d = q.shape[-1]
        out = np.zeros((len(rows), d))
        lse = np.zeros(len(rows))
        for r, (b, h, i) in enumerate(rows):
            K, V = np.asarray(k[b, h], float), np.asarray(v[b, h], float)
            Q = np.asarray(q[b, h][i], float)
            if kind == "transposed_kv":
                K, V = V, K
            s = (Q @ K.T) * (1.0 if kind == "no_scale" else scale)
            j = np.arange(K.shape[0])
            if causal:
                allowed = (j < i) | (j == 0) if kind == "strict_mask" else j <= i
                s = np.where(allowed, s, -np.inf)
            m = s.max()
            if kind == "no_max_sub":
                w = np.exp(s)
                m = 0.0
            elif kind == "wrong_sign":
                w = np.exp(m - s)
            else:
                w = np.exp(s - m)
            z = w.sum()
            if kind == "drop_last_key" and K.shape[0] > 1:
                z = w[:-1].sum()
            out[r] = (w @ V) / z
            lse[r] = (np.log(z)) if kind == "lse_without_max" else m + np.log(z)
        return out, lse
    return impl


def test_pins_accept_the_oracle():
    assert _pin_failures(attention_rows) == []
    assert _pin_failures(lambda *a: online_attention_rows(*a, tile=2)) == []


@pytest.mark.parametrize("kind", ["transposed_kv", "no_scale", "strict_mask", "no_max_sub",
                                  "wrong_sign", "drop_last_key", "lse_without_max"])
def test_pins_reject_planted_mistakes(kind):
    import warnings
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", RuntimeWarning)
        fails = _pin_failures(_mutant(kind))
    assert fails, f"mutant {kind} passed every pin"


def test_pins_reject_merge_without_rescale():
    """A merge that forgets to rescale the accumulator fails the block pins."""
    import oracle.attention as A

    real = A.merge_block

    def bad(m, total, acc, scores, values):
        new_m, new_total, new_acc = real(m, total, acc, scores, values)
        with np.errstate(invalid="ignore"):
            old = np.where(np.isneginf(m), 0.0, np.exp(m - new_m))
        # undo the accumulator rescale only: acc + w V instead of a acc + w V
        return new_m, new_total, new_acc + acc * (1 - old[:, None])

    A.merge_block = bad
    try:
        fails = _pin_failures(lambda *a: A.online_attention_rows(*a, tile=2))
    finally:
        A.merge_block = real
    assert fails


# ---------------------------------------------------------------------------
# Partial states over key ranges, and their merge
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_key_range_states_is_full_attention(causal):
    """Attention over disjoint key ranges, merged, equals attention over all keys."""
    from oracle import merge_states

    rng = np.random.default_rng(11)
    B, H, N, d = 1, 2, 300, 8
    q = rng.standard_normal((B, H, N, d)) * 2
    k = rng.standard_normal((B, H, N, d))
    v = rng.standard_normal((B, H, N, d))
    rows = all_rows(B, H, N)
    full_o, full_l = attention_rows(q, k, v, 0.4, causal, rows)
    bounds = [0, 1, 128, 129, 256, 300]
    parts = [attention_rows(q, k, v, 0.4, causal, rows, key_range=(lo, hi))
             for lo, hi in zip(bounds[:-1], bounds[1:])]
    o, l = merge_states([p[0] for p in parts], [p[1] for p in parts])
    assert np.allclose(o, full_o, rtol=1e-12, atol=1e-13)
    assert np.allclose(l, full_l, rtol=1e-12, atol=1e-13)
    # the order of the states does not matter
    o2, l2 = merge_states([p[0] for p in parts[::-1]], [p[1] for p in parts[::-1]])
    assert np.allclose(o2, full_o, rtol=1e-12, atol=1e-13)
    if causal:
        # rows before a range's first key have an empty state there
        assert np.isneginf(parts[-1][1][:256]).all() and (parts[-1][0][:256] == 0).all()


def test_key_range_state_closed_form():
    """One key in range: the state is that key's value and its score."""
    q, k, v = scalar_problem([0.0, 1.0, 2.0], [10.0, 20.0, 30.0])
    o, l = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, 3), key_range=(1, 2))
    assert (o[:, 0] == 20.0).all() and (l == 1.0).all()
    o, l = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, 3), key_range=(3, 3))
    assert (o == 0).all() and np.isneginf(l).all()


def test_merge_rejects_missing_rescale():
    """A merge that does not rescale the old accumulator is caught by the pin."""
    from oracle import merge_states

    q, k, v = scalar_problem([0.0, 1.0, 2.0], [10.0, 20.0, 30.0])
    rows = all_rows(1, 1, 3)
    parts = [attention_rows(q, k, v, 1.0, False, rows, key_range=(lo, lo + 1)) for lo in range(3)]
    o, _ = merge_states([p[0] for p in parts], [p[1] for p in parts])
    assert round(o[0, 0], 6) == 25.752104
    # planted mistake: plain average of the partial outputs (block averaging)
    bad = np.mean([p[0] for p in parts], axis=0)
    assert abs(bad[0, 0] - o[0, 0]) > 1.0


# ---------------------------------------------------------------------------
# Backward: gradients of L = sum(O * dO)
# ---------------------------------------------------------------------------

def _loss(q, k, v, do, scale, causal):
    o, _ = attention_full(q, k, v, scale, causal)
    return float((o * do).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    from oracle import attention_backward

    rng = np.random.default_rng(31 + int(causal))
    B, H, N, d = 1, 2, 6, 3
    q, k, v, do = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    scale = 0.8
    dq, dk, dv, _ = attention_backward(q, k, v, do, scale, causal)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            num[idx] = (lp - lm) / (2 * eps)
        assert np.allclose(g, num, rtol=1e-6, atol=1e-8), name


def test_backward_closed_forms():
    from oracle import attention_backward

    rng = np.random.default_rng(8)
    B, H, N, d = 1, 1, 7, 4
    q = rng.standard_normal((B, H, N, d))
    k = np.broadcast_to(rng.standard_normal((1, 1, 1, d)), (B, H, N, d)).copy()
    v = rng.standard_normal((B, H, N, d))
    do = rng.standard_normal((B, H, N, d))
    for causal in (False, True):
        dq, dk, dv, D = attention_backward(q, k, v, do, 0.6, causal)
        # all keys equal: every score row is constant, so dQ = 0 exactly
        assert np.allclose(dq, 0.0, atol=1e-13)
        # uniform weights: dV_j = sum over queries that see j of dO_i / (#keys they see)
        n_allowed = np.arange(1, N + 1) if causal else np.full(N, N)
        for j in range(N):
            rows = [i for i in range(N) if (not causal or j <= i)]
            expect = sum(do[0, 0, i] / n_allowed[i] for i in rows)
            assert np.allclose(dv[0, 0, j], expect, atol=1e-13)
    # D = rowsum(dO * O) equals rowsum(P * dP): check against the forward
    o, _ = attention_full(q, k, v, 0.6, False)
    _, _, _, D = attention_backward(q, k, v, do, 0.6, False)
    assert np.allclose(D, (o * do).sum(-1), rtol=1e-13)


def test_backward_pins_reject_a_dropped_term():
    """Leaving D out of dS is caught by the finite-difference pin."""
    from oracle import attention_backward

    rng = np.random.default_rng(2)
    q, k, v, do = (rng.standard_normal((1, 1, 5, 3)) for _ in range(4))
    dq, dk, dv, D = attention_backward(q, k, v, do, 1.0, False)
    # rebuild dQ without the D term
    S = q[0, 0] @ k[0, 0].T
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    bad_dq = (P * (do[0, 0] @ v[0, 0].T)) @ k[0, 0]
    eps = 1e-6
    qp, qm = q.copy(), q.copy()
    qp[0, 0, 2, 1] += eps
    qm[0, 0, 2, 1] -= eps
    num = (_loss(qp, k, v, do, 1.0, False) - _loss(qm, k, v, do, 1.0, False)) / (2 * eps)
    assert abs(dq[0, 0, 2, 1] - num) < 1e-7
    assert abs(bad_dq[2, 1] - num) > 1e-3


# ---------------------------------------------------------------------------
# Block-sparse attention: the softmax over the key blocks a layout retains
# ---------------------------------------------------------------------------

def _random_layout(rng, nqb, nkb, density=0.5):
    lay = rng.random((nqb, nkb)) < density
    lay[0, :] = False  # one query block with no key at all
    return lay


@pytest.mark.parametrize("seed", range(8))
def test_block_sparse_brute_force_tiny(seed):
    """Random block layouts (one row block empty) against pure-Python loops."""
    from oracle import block_sparse_attention_rows

    rng = np.random.default_rng(300 + seed)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
    N, d = int(rng.integers(5, 18)), int(rng.integers(1, 6))
    bq, bk = int(rng.integers(1, 5)), int(rng.integers(1, 5))
    lay = _random_layout(rng, -(-N // bq), -(-N // bk))
    q = rng.standard_normal((B, H, N, d))
    k = rng.standard_normal((B, H, N, d))
    v = rng.standard_normal((B, H, N, d))
    causal = bool(seed % 2)
    bo, bl = brute_force_attention(q, k, v, 0.7, causal, layout=lay, block_q=bq, block_k=bk)
    o, l = block_sparse_attention_rows(q, k, v, 0.7, causal, all_rows(B, H, N), lay, bq, bk)
    assert np.allclose(o, np.array(bo).reshape(o.shape), rtol=1e-12, atol=1e-13)
    bl = np.array(bl).reshape(l.shape)
    assert (np.isneginf(l) == np.isneginf(bl)).all()
    fin = np.isfinite(bl)
    assert np.allclose(l[fin], bl[fin], rtol=1e-12, atol=1e-13)
    # the empty first query block: O = 0, LSE = -inf
    first = all_rows(B, H, N)[:, 2] < bq
    assert (o[first] == 0).all() and np.isneginf(l[first]).all()


def test_block_sparse_full_layout_is_dense_and_block_diagonal_is_per_block():
    """All blocks retained = dense attention; a block-diagonal layout = each block alone."""
    from oracle import block_sparse_attention_rows

    rng = np.random.default_rng(21)
    B, H, N, d = 1, 2, 96, 8
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    rows = all_rows(B, H, N)
    dense_o, dense_l = attention_rows(q, k, v, 0.5, True, rows)
    o, l = block_sparse_attention_rows(q, k, v, 0.5, True, rows, np.ones((3, 6), bool), 32, 16)
    assert np.allclose(o, dense_o, rtol=1e-13, atol=1e-14) and np.allclose(l, dense_l, rtol=1e-13)
    # block-diagonal with 32-row and 32-key blocks: three independent problems
    o, l = block_sparse_attention_rows(q, k, v, 0.5, False, rows, np.eye(3, dtype=bool), 32, 32)
    o = o.reshape(B, H, N, d)
    l = l.reshape(B, H, N)
    for blk in range(3):
        sl = slice(32 * blk, 32 * blk + 32)
        bo, bl = attention_full(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.5, False)
        assert np.allclose(o[:, :, sl], bo, rtol=1e-12, atol=1e-13)
        assert np.allclose(l[:, :, sl], bl, rtol=1e-12, atol=1e-13)


def test_block_sparse_single_block_closed_form():
    """One retained key block whose values all equal c: O = c, LSE = logsumexp of its scores."""
    from oracle import block_sparse_attention_rows

    N, d = 12, 3
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, N, d))
    k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, d))
    v[0, 0, 4:8] = [1.5, -2.0, 0.25]
    lay = np.zeros((3, 3), bool)
    lay[:, 1] = True  # keys 4..7 only
    o, l = block_sparse_attention_rows(q, k, v, 1.0, False, all_rows(1, 1, N), lay, 4, 4)
    assert np.allclose(o, [1.5, -2.0, 0.25], rtol=1e-14)
    s = q[0, 0] @ k[0, 0, 4:8].T
    assert np.allclose(l, np.log(np.exp(s).sum(axis=1)), rtol=1e-13)


def test_block_sparse_pins_reject_a_transposed_layout():
    """A mutant that indexes the layout as [key block, query block] fails the brute-force pin."""
    rng = np.random.default_rng(77)
    N, d, bq, bk = 12, 2, 3, 4
    lay = np.zeros((4, 3), bool)
    lay[3, 0] = lay[1, 2] = lay[0, 0] = lay[2, 1] = True
    q, k, v = (rng.standard_normal((1, 1, N, d)) for _ in range(3))
    lay_t = lambda b, h, i, j: lay.T[np.minimum(np.asarray(i)[:, None] // bk, 2),
                                     np.minimum(np.asarray(j)[None, :] // bq, 3)]
    bad_o, _ = attention_rows(q, k, v, 1.0, False, all_rows(1, 1, N), key_mask=lay_t)
    bo, _ = brute_force_attention(q, k, v, 1.0, False, layout=lay, block_q=bq, block_k=bk)
    assert not np.allclose(bad_o, np.array(bo).reshape(bad_o.shape), atol=1e-6)


def test_block_layout_from_csr():
    from oracle import block_layout_from_csr

    lay = block_layout_from_csr([0, 2, 2, 3], [0, 3, 1], 4)
    assert lay.tolist() == [[True, False, False, True], [False] * 4, [False, True, False, False]]
