"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no attention arithmetic: it only draws random tensors and
picks row samples.  Both the CUDA path and the oracle are fed from here.

Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws Q, K, V in that
order with ``torch.randn(B, H, N, d)`` in float32; Q is multiplied by
``q_std``; all three are rounded to bfloat16 (round to nearest even).  The
oracle reads the bfloat16 values, widened exactly.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One attention-forward problem: shapes, mask, scale and input seed."""

    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    q_std: float = 1.0
    sample_rows: int = 0  # 0 = every row is checked against the oracle

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """4*B*H*N^2*d, halved for causal (the counting convention)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def as_config(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "H": self.H, "N": self.N,
            "d": self.d, "causal": self.causal, "seed": self.seed,
            "q_std": self.q_std, "scale": self.scale,
        }


# The five problems of the benchmark plan, named by their shape.
WORKLOADS = {
    w.name: w
    for w in (
        Workload("b1h1n256d64", 1, 1, 256, 64, False, 0),
        Workload("b4h16n4096d64", 4, 16, 4096, 64, False, 1, sample_rows=4096),
        Workload("b2h16n8192d128_causal", 2, 16, 8192, 128, True, 2, sample_rows=4096),
        Workload("b1h32n32768d128_causal_q4", 1, 32, 32768, 128, True, 3, q_std=4.0,
                 sample_rows=2048),
        Workload("b1h8n131072d128_causal", 1, 8, 131072, 128, True, 4, sample_rows=1024),
        # few query blocks for 148 SMs: the shapes the split-KV path is for
        Workload("b1h2n8192d128", 1, 2, 8192, 128, False, 5, sample_rows=1024),
        Workload("b1h1n32768d128_causal", 1, 1, 32768, 128, True, 6, sample_rows=1024),
        # small enough for multi-pass ncu captures of the materialising comparator
        Workload("b1h4n4096d128_causal", 1, 4, 4096, 128, True, 7, sample_rows=1024),
        # four of the eight heads of the N = 131072 causal problem: the same
        # long-context work list at half the size, for multi-pass ncu captures
        Workload("b1h4n131072d128_causal", 1, 4, 131072, 128, True, 8, sample_rows=1024),
    )
}


def make_qkv(B: int, H: int, N: int, d: int, seed: int, q_std: float = 1.0,
             k_std: float = 1.0, v_std: float = 1.0):
    """Q, K, V as contiguous CPU bfloat16 tensors [B, H, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q.mul_(q_std)
    if k_std != 1.0:
        k.mul_(k_std)
    if v_std != 1.0:
        v.mul_(v_std)
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def make_workload_inputs(w: Workload):
    return make_qkv(w.B, w.H, w.N, w.d, w.seed, w.q_std)


def sample_rows(B: int, H: int, N: int, count: int, seed: int) -> torch.Tensor:
    """Rows (b, h, i) to check: ``count`` random ones plus forced edge rows.

    The random rows come from ``torch.randperm`` with generator seed
    1000 + seed; the forced rows are i in {0, 1, 127, 128, N-1} (those that
    exist) for h in {0, H-1}, b in {0, B-1}.  ``count <= 0`` returns every row.
    """
    total = B * H * N
    if count <= 0 or count >= total:
        idx = torch.arange(total)
    else:
        g = torch.Generator(device="cpu").manual_seed(1000 + int(seed))
        idx = torch.randperm(total, generator=g)[:count]
        forced = []
        for b in sorted({0, B - 1}):
            for h in sorted({0, H - 1}):
                for i in (0, 1, 127, 128, N - 1):
                    if 0 <= i < N:
                        forced.append((b * H + h) * N + i)
        idx = torch.unique(torch.cat([idx, torch.tensor(forced, dtype=torch.long)]))
    b = idx // (H * N)
    h = (idx // N) % H
    i = idx % N
    return torch.stack([b, h, i], dim=1)


def make_local_qkv(B: int, H: int, N: int, d: int, seed: int, length_scale: float = 64.0,
                   peak: float = 10.0):
    """Q, K, V (CPU bf16 [B, H, N, d]) whose scores fall off with distance.

    Half of each head's width carries random Fourier features of the
    position: F = d/4 frequencies w ~ N(0, 1/length_scale^2) per head, a
    cosine and a sine of w*i each, the same features in Q and K.  Their dot
    product is a^2 sum_f cos(w_f (i - j)), whose mean over the frequencies is
    a^2 F exp(-(i-j)^2 / (2 length_scale^2)); a is set so that, with the
    scale 1/sqrt(d), this positional score is ``peak`` at distance 0.  The
    other half of Q and K, and all of V, is N(0, 1).  Attention then
    concentrates near the diagonal, the case where a block-sparse layout
    that keeps a band of key blocks can match exact attention.

    Recipe: a CPU generator seeded with ``seed`` draws the frequencies
    [B, H, F], then the Q content, K content and V (float32 randn, in that
    order); the features are computed in float64; everything is rounded to
    bfloat16 at the end.
    """
    if d % 4:
        raise ValueError("d must be a multiple of 4")
    F = d // 4
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    w = torch.randn((B, H, F), generator=g, dtype=torch.float64) / float(length_scale)
    qc = torch.randn((B, H, N, d // 2), generator=g, dtype=torch.float32)
    kc = torch.randn((B, H, N, d // 2), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, N, d), generator=g, dtype=torch.float32)
    a = math.sqrt(peak * math.sqrt(d) / F)
    ang = torch.arange(N, dtype=torch.float64)[None, None, :, None] * w[:, :, None, :]
    feat = (a * torch.cat([torch.cos(ang), torch.sin(ang)], dim=-1)).to(torch.float32)
    q = torch.cat([feat, qc], dim=-1)
    k = torch.cat([feat, kc], dim=-1)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def local_block_layout(N: int, window: int, causal: bool, block_q: int, block_k: int,
                       sinks: int = 0):
    """Band layout: bool [ceil(N/block_q), ceil(N/block_k)] as nested lists.

    Query block r retains key block c when c's keys meet the rows of r widened
    by ``window`` keys to the left (and, unless causal, to the right), or when
    c < ``sinks`` (the first key blocks, kept for every query block).
    """
    nqb, nkb = -(-N // block_q), -(-N // block_k)
    lay = []
    for r in range(nqb):
        lo = r * block_q - window
        hi = min(N, (r + 1) * block_q) - 1 + (0 if causal else window)
        lay.append([(c < sinks) or (c * block_k <= hi and (c + 1) * block_k - 1 >= lo)
                    for c in range(nkb)])
    return lay
