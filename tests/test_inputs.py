"""Host logic of the seeded input generators (no GPU, no attention arithmetic)."""

import torch

from exact_softmax_attention_02_b200.inputs import WORKLOADS, make_qkv, sample_rows


def test_make_qkv_is_seeded_and_bf16():
    a = make_qkv(1, 2, 16, 8, seed=3)
    b = make_qkv(1, 2, 16, 8, seed=3)
    c = make_qkv(1, 2, 16, 8, seed=4)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    # Q, K, V are drawn in that order from one generator
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 2, 16, 8, generator=g)
    k = torch.randn(1, 2, 16, 8, generator=g)
    assert torch.equal(a[0], q.to(torch.bfloat16)) and torch.equal(a[1], k.to(torch.bfloat16))


def test_q_std_scales_queries_only():
    base = make_qkv(1, 1, 32, 16, seed=3)
    big = make_qkv(1, 1, 32, 16, seed=3, q_std=4.0)
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 1, 32, 16, generator=g)
    assert torch.equal(big[0], (q * 4.0).to(torch.bfloat16))
    assert torch.equal(big[1], base[1]) and torch.equal(big[2], base[2])


def test_sample_rows_forced_and_unique():
    rows = sample_rows(2, 3, 300, 50, seed=1)
    assert rows.shape[1] == 3
    keyed = (rows[:, 0] * 3 + rows[:, 1]) * 300 + rows[:, 2]
    assert len(torch.unique(keyed)) == len(keyed)
    for b in (0, 1):
        for h in (0, 2):
            for i in (0, 1, 127, 128, 299):
                assert ((rows[:, 0] == b) & (rows[:, 1] == h) & (rows[:, 2] == i)).any()
    assert torch.equal(rows, sample_rows(2, 3, 300, 50, seed=1))
    full = sample_rows(1, 2, 10, 0, seed=0)
    assert full.shape[0] == 20


def test_workload_flop_counts():
    w = WORKLOADS["b2h16n8192d128_causal"]
    assert w.flops == 4 * 2 * 16 * 8192 ** 2 * 128 / 2
    w = WORKLOADS["b4h16n4096d64"]
    assert w.flops == 4 * 4 * 16 * 4096 ** 2 * 64
    assert abs(w.scale - 0.125) < 1e-15
