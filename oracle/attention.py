"""Float64 CPU oracle for exact softmax attention (forward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA
path (no kernels, headers, helpers or constants) and imports nothing from the
package.

What it computes
----------------
For every selected query row i of head (b, h):

    s_j   = scale * <Q[b,h,i,:], K[b,h,j,:]>      for allowed keys j
    M     = max_j s_j
    w_j   = exp(s_j - M)
    Z     = sum_j w_j
    O_i   = (sum_j w_j V[b,h,j,:]) / Z
    LSE_i = M + ln Z

This is the dense-attention definition O = softmax(Q K^T / sqrt(d)) V of
"FlashAttention: the intermediate matrix comes first" (lihaoran.work, the
opening formula), evaluated with the max-subtracted full-weight softmax that
the pages use as their reference: liminalml.com "FlashAttention", the
executable scalar example (weights relative to the largest score, weighted sum
over their total), and lihaoran.work "Check three scores" (the full-weight
``reference`` function).  The allowed keys are all j, or j <= i when causal
(reading: the pages only name "causal masking"; query and key sequences have
the same length, so the diagonal is always allowed and no row is empty).
LSE is the natural-log log-sum-exp of the scaled scores (reading: the pages
keep m and the denominator but never name LSE).

Three functions, three independent computations:

* ``attention_rows``    -- the definition above, one full score row at a time.
* ``online_attention_rows`` -- the tile-wise online recurrence with running
  (m, total, acc), merged block by block (interactiveml.org "FlashAttention
  saves the matrix, not the quadratic work", the vector-valued block merge
  with the guard for m = -inf; liminalml.com "FlashAttention", the block
  update m' = max(m, max s), a = e^(m-m'), p = e^(s-m'), l' = a l + sum p,
  u' = a u + p V, output u / l).  Tile width 64, as in the 64-by-64 score
  tile of the interactiveml.org page.
* ``brute_force_attention`` -- pure-Python loops, no max subtraction, exact
  summation with ``math.fsum``; only for tiny inputs.

``attention_backward`` gives dQ, dK, dV of L = sum(O * dO), the derivative
of the same definition (pinned by finite differences).

``block_sparse_attention_rows`` restricts the allowed keys to the blocks a
block layout retains (the block-sparse comparison the pages suggest).

``attention_rows(..., key_range=(lo, hi))`` gives the partial state of one
key range, and ``merge_states`` folds such states together (the block update
applied to whole states); merged states over disjoint ranges equal the full
row (pinned in tests/test_oracle_pins.py).

Inputs are arrays of shape [B, H, N, d] of any real dtype (bf16 values
widened to float32 or float64 are exact); they are converted to float64 here.

Parity pins (tests/test_oracle_pins.py) tie every function to the pages'
worked examples, closed forms, invariants and brute force.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "attention_rows",
    "attention_backward",
    "merge_states",
    "attention_full",
    "block_sparse_attention_rows",
    "block_layout_from_csr",
    "online_attention_rows",
    "merge_block",
    "brute_force_attention",
    "scalar_softmax_weighted_sum",
    "scalar_online_weighted_sum",
    "flops_for_rows",
]

# Bound on the float64 score block held at once (rows x keys).
_MAX_BLOCK_ELEMS = 1 << 24


def _as_f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _group_rows(rows: np.ndarray):
    """Yield (b, h, positions, query indices) for each head that has rows."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    if rows.shape[0] == 0:
        return
    key = rows[:, 0] * (1 << 40) + rows[:, 1] * (1 << 20)
    order = np.argsort(key, kind="stable")
    sorted_key = key[order]
    starts = np.flatnonzero(np.r_[True, sorted_key[1:] != sorted_key[:-1]])
    ends = np.r_[starts[1:], len(order)]
    for s, e in zip(starts, ends):
        pos = order[s:e]
        b, h = int(rows[pos[0], 0]), int(rows[pos[0], 1])
        yield b, h, pos, rows[pos, 2]


def attention_rows(q, k, v, scale: float, causal: bool, rows, key_range=None, key_mask=None):
    """Exact attention output and LSE for the selected rows.

    Follows the dense definition O = softmax(scale * Q K^T) V
    (lihaoran.work, "The intermediate matrix comes first") with the
    max-subtracted full-weight softmax of the pages' reference examples
    (liminalml.com "FlashAttention", the scalar example; lihaoran.work
    "Check three scores").

    Args:
      q, k, v: arrays [B, H, N, d].
      scale:   multiplier of the dot product (1/sqrt(d) by default upstream).
      causal:  if true, query i sees keys j <= i only.
      rows:    int array [R, 3] of (b, h, i).
      key_range: optional (lo, hi): only keys lo <= j < hi are allowed (the
               partial state of one key range).  A row with no allowed key
               gets O = 0 and LSE = -inf (the empty state, weight 0 in a merge).
      key_mask: optional callable (b, h, i [r], j [N]) -> bool [r, N]; keys
               where it is false are not allowed (block-sparse retention).

    Returns:
      (O, LSE): float64 arrays [R, d] and [R].
    """
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    d = q.shape[-1]
    n_keys = k.shape[2]
    out = np.zeros((rows.shape[0], d), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    for b, h, pos, qi in _group_rows(rows):
        K = _as_f64(k[b, h])  # [N, d]
        V = _as_f64(v[b, h])  # [N, d]
        chunk = max(1, _MAX_BLOCK_ELEMS // max(1, n_keys))
        for c0 in range(0, len(pos), chunk):
            p = pos[c0:c0 + chunk]
            i = qi[c0:c0 + chunk]
            Q = _as_f64(q[b, h][i])  # [r, d]
            s = scale * (Q @ K.T)  # [r, N]   the score rows
            j = np.arange(n_keys)
            if causal:
                s = np.where(j[None, :] <= i[:, None], s, -np.inf)
            if key_range is not None:
                lo, hi = key_range
                s = np.where((j[None, :] >= lo) & (j[None, :] < hi), s, -np.inf)
            if key_mask is not None:
                s = np.where(key_mask(b, h, i, j), s, -np.inf)
            m = s.max(axis=1)  # largest score of each row
            empty = np.isneginf(m)
            m_safe = np.where(empty, 0.0, m)
            w = np.exp(s - m_safe[:, None])  # weights relative to it; masked -> 0
            z = w.sum(axis=1)  # denominator
            with np.errstate(invalid="ignore", divide="ignore"):
                out[p] = np.where(empty[:, None], 0.0, (w @ V) / z[:, None])
                lse[p] = np.where(empty, -np.inf, m + np.log(z))
    return out, lse


def attention_full(q, k, v, scale: float, causal: bool):
    """All rows of ``attention_rows``, reshaped to [B, H, N, d] and [B, H, N]."""
    B, H, N, d = q.shape
    b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), indexing="ij")
    rows = np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1)
    o, l = attention_rows(q, k, v, scale, causal, rows)
    return o.reshape(B, H, N, d), l.reshape(B, H, N)


def block_sparse_attention_rows(q, k, v, scale: float, causal: bool, rows, layout,
                                block_q: int, block_k: int):
    """Attention restricted to the key blocks a block layout retains.

    The pages treat sparsity as a separate design dimension that decides which
    query-key interactions are kept (liminalml.com "FlashAttention", the
    question "Is it sparse attention?"), and suggest comparing exact and
    block-sparse attention at matched output error (interactiveml.org
    "FlashAttention saves the matrix, not the quadratic work", the suggested
    experiments).  Reading: block-sparse attention is the same softmax over a
    smaller allowed set.  Query i may see key j only if
    layout[i // block_q, j // block_k] is set (and j <= i when causal).  A
    query with no allowed key gets O = 0 and LSE = -inf.

    Args:
      layout: bool array [ceil(N / block_q), ceil(N / block_k)], shared by
              every (b, h).
      block_q, block_k: query rows and keys per block.
    Other arguments and the return value as in ``attention_rows``.
    """
    lay = np.asarray(layout, dtype=bool)

    def mask(b, h, i, j):
        return lay[np.asarray(i)[:, None] // block_q, np.asarray(j)[None, :] // block_k]

    return attention_rows(q, k, v, scale, causal, rows, key_mask=mask)


def block_layout_from_csr(row_ptr, col_idx, n_kblocks: int) -> np.ndarray:
    """Dense bool layout [len(row_ptr) - 1, n_kblocks] from CSR block lists.

    Row r retains key blocks col_idx[row_ptr[r]:row_ptr[r+1]].
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    col_idx = np.asarray(col_idx, dtype=np.int64)
    lay = np.zeros((len(row_ptr) - 1, n_kblocks), dtype=bool)
    for r in range(len(row_ptr) - 1):
        lay[r, col_idx[row_ptr[r]:row_ptr[r + 1]]] = True
    return lay


def merge_block(m, total, acc, scores, values):
    """Fold one block of scores into the running statistics of each row.

    The three sufficient statistics of interactiveml.org ("FlashAttention
    saves the matrix, not the quadratic work"): the largest score so far m,
    the rescaled exponential sum, and the rescaled weighted-value
    accumulator.  A larger block maximum rescales both the sum and the
    accumulator by one factor exp(m - m_new) (liminalml.com, the block update
    and the 5 -> 10 question); the factor is 0 while m is still -inf.

    Args (R rows, T keys in the block, d value width):
      m:      [R] running max (-inf before the first key).
      total:  [R] running denominator.
      acc:    [R, d] running unnormalised numerator.
      scores: [R, T] scores of the block (-inf = masked key).
      values: [T, d] value rows of the block.
    Returns updated (m, total, acc).
    """
    block_max = scores.max(axis=1)
    new_max = np.maximum(m, block_max)
    with np.errstate(invalid="ignore"):
        old_scale = np.where(np.isneginf(m), 0.0, np.exp(m - new_max))
        # A row whose max is still -inf has seen no allowed key: weight 0.
        weight = np.where(np.isneginf(new_max)[:, None], 0.0,
                          np.exp(scores - new_max[:, None]))
    total = total * old_scale + weight.sum(axis=1)
    acc = acc * old_scale[:, None] + weight @ values
    return new_max, total, acc


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Gradients of L = sum(O * dO) with O = softmax(scale Q K^T [mask]) V.

    The pages name the backward pass only ("selected recomputation in the
    backward pass", lihaoran.work; "tiling, fusion, and recomputation",
    liminalml.com "Why use it?").  What it computes is the derivative of the
    forward definition, written out per head with the full score matrix:

        P  = softmax(scale * Q K^T) over the allowed keys
        dV = P^T dO
        dP = dO V^T
        D  = rowsum(dO * O)          (= rowsum(P * dP))
        dS = P * (dP - D)
        dQ = scale * dS K
        dK = scale * dS^T Q

    Args: q, k, v, do arrays [B, H, N, d].  Returns float64 (dQ, dK, dV, D),
    D of shape [B, H, N].
    """
    B, H, N, d = np.shape(q)
    dq = np.zeros((B, H, N, d))
    dk = np.zeros((B, H, N, d))
    dv = np.zeros((B, H, N, d))
    dd = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            Q, K, V, dO = (_as_f64(t[b, h]) for t in (q, k, v, do))
            S = scale * (Q @ K.T)
            if causal:
                S = np.where(np.tril(np.ones((N, N), dtype=bool)), S, -np.inf)
            M = S.max(axis=1, keepdims=True)
            W = np.exp(S - M)
            P = W / W.sum(axis=1, keepdims=True)
            O = P @ V
            dv[b, h] = P.T @ dO
            dP = dO @ V.T
            D = (dO * O).sum(axis=1)
            dS = P * (dP - D[:, None])
            dq[b, h] = scale * (dS @ K)
            dk[b, h] = scale * (dS.T @ Q)
            dd[b, h] = D
    return dq, dk, dv, dd


def merge_states(o_parts, lse_parts):
    """Merge partial attention states of the same rows over disjoint key ranges.

    Each state s is a normalised partial output O_s = u_s / l_s and its
    log-sum-exp LSE_s = m_s + ln l_s.  Folding them in one after another is
    the block update with whole states as blocks (liminalml.com
    "FlashAttention": m' = max(m, m_s), both the running numerator and
    denominator rescaled by e^(m - m'); interactiveml.org: the old scale is 0
    while m = -inf).  An empty state (LSE = -inf) has weight 0.

    Args: o_parts [S, R, d], lse_parts [S, R].  Returns (O [R, d], LSE [R]).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.full(lse_parts.shape[1], -np.inf)
    total = np.zeros(lse_parts.shape[1])
    acc = np.zeros(o_parts.shape[1:])
    with np.errstate(invalid="ignore"):
        for o_s, l_s in zip(o_parts, lse_parts):
            new_m = np.maximum(m, l_s)
            old_scale = np.where(np.isneginf(m), 0.0, np.exp(m - new_m))
            weight = np.where(np.isneginf(l_s), 0.0, np.exp(l_s - np.where(np.isneginf(new_m), 0.0, new_m)))
            total = total * old_scale + weight
            acc = acc * old_scale[:, None] + weight[:, None] * o_s
            m = new_m
        out = np.where(total[:, None] > 0, acc / np.where(total > 0, total, 1.0)[:, None], 0.0)
        lse = np.where(total > 0, m + np.log(np.where(total > 0, total, 1.0)), -np.inf)
    return out, lse


def online_attention_rows(q, k, v, scale: float, causal: bool, rows, tile: int = 64):
    """The same rows computed by the tile-wise online recurrence.

    Keys are visited in tiles of ``tile`` (64 as in the interactiveml.org
    64-by-64 score tile); each tile is folded in with ``merge_block``; the
    output is acc / total and LSE = m + ln(total) (liminalml.com
    "FlashAttention": after the final block, output u / l).
    """
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    d = q.shape[-1]
    n_keys = k.shape[2]
    out = np.zeros((rows.shape[0], d), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    for b, h, pos, qi in _group_rows(rows):
        K = _as_f64(k[b, h])
        V = _as_f64(v[b, h])
        Q = _as_f64(q[b, h][qi])
        r = len(pos)
        m = np.full(r, -np.inf)
        total = np.zeros(r)
        acc = np.zeros((r, d))
        for j0 in range(0, n_keys, tile):
            j = np.arange(j0, min(j0 + tile, n_keys))
            s = scale * (Q @ K[j].T)
            if causal:
                s = np.where(j[None, :] <= qi[:, None], s, -np.inf)
            m, total, acc = merge_block(m, total, acc, s, V[j])
        out[pos] = acc / total[:, None]
        lse[pos] = m + np.log(total)
    return out, lse


def brute_force_attention(q, k, v, scale: float, causal: bool, layout=None, block_q: int = 1,
                          block_k: int = 1):
    """Pure-Python softmax attention without max subtraction (tiny inputs).

    O_i = sum_j e^{s_ij} V_j / sum_j e^{s_ij}, summed exactly with
    math.fsum; LSE_i = ln sum_j e^{s_ij}.  Only valid while every e^{s}
    is representable, i.e. for small scores.  With a block layout (nested
    lists or array of booleans), key j is skipped for query i unless
    layout[i // block_q][j // block_k] is set; a query left with no key gets
    O = 0 and LSE = -inf.  Returns nested lists O[b][h][i][c] and LSE[b][h][i].
    """
    B, H, N, d = (int(x) for x in np.shape(q))
    qf, kf, vf = (np.asarray(t, dtype=np.float64).tolist() for t in (q, k, v))
    O = [[[[0.0] * d for _ in range(N)] for _ in range(H)] for _ in range(B)]
    L = [[[0.0] * N for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(N):
                e = []
                for j in range(N):
                    if causal and j > i:
                        continue
                    if layout is not None and not layout[i // block_q][j // block_k]:
                        continue
                    s = scale * math.fsum(qf[b][h][i][c] * kf[b][h][j][c] for c in range(d))
                    e.append((j, math.exp(s)))
                if not e:
                    L[b][h][i] = -math.inf
                    continue
                z = math.fsum(w for _, w in e)
                for c in range(d):
                    O[b][h][i][c] = math.fsum(w * vf[b][h][j][c] for j, w in e) / z
                L[b][h][i] = math.log(z)
    return O, L


def scalar_softmax_weighted_sum(scores, values):
    """Full-weight softmax average of scalar values (the pages' reference).

    Weights are e^{s - max s}; the result is sum(w v) / sum(w)
    (liminalml.com "FlashAttention" scalar example; lihaoran.work "Check
    three scores").  Returns (output, lse).
    """
    mx = max(scores)
    w = [math.exp(s - mx) for s in scores]
    z = math.fsum(w)
    return math.fsum(wi * vi for wi, vi in zip(w, values)) / z, mx + math.log(z)


def scalar_online_weighted_sum(scores, values, block: int = 1):
    """One pass over scalar (score, value) pairs with running statistics.

    Per block: m' = max(m, max block), old terms rescaled by e^{m - m'},
    new terms weighted e^{s - m'} (lihaoran.work, the one-item recurrence
    l' = e^{m-m'} l + e^{a-m'}, u' = e^{m-m'} u + e^{a-m'} v; with block > 1
    the liminalml.com block update).  Returns (output, lse).
    """
    m, total, weighted = -math.inf, 0.0, 0.0
    for start in range(0, len(scores), block):
        blk_s = scores[start:start + block]
        blk_v = values[start:start + block]
        new_m = max(m, max(blk_s))
        old = 0.0 if m == -math.inf else math.exp(m - new_m)
        total *= old
        weighted *= old
        for s, val in zip(blk_s, blk_v):
            w = math.exp(s - new_m)
            total += w
            weighted += w * val
        m = new_m
    return weighted / total, m + math.log(total)


def flops_for_rows(rows, n_keys: int, d: int, causal: bool) -> float:
    """Multiply-add count x 2 of the two products for the given rows.

    Each allowed (query, key) pair costs d multiply-adds for the score and d
    for the weighted value sum (interactiveml.org: roughly 2 N^2 d
    multiply-adds per head), i.e. 4 d FLOPs.
    """
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    if causal:
        allowed = np.minimum(rows[:, 2] + 1, n_keys).astype(np.float64).sum()
    else:
        allowed = float(rows.shape[0]) * n_keys
    return 4.0 * d * allowed
