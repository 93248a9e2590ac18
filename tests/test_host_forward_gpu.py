"""The host-buffer forward (fa_fwd_host): copies pipelined with the kernels.

Every (b, h) pair is computed by the same kernel whatever the grouping of
heads, so the host path must give fa_fwd's result bit for bit, for any number
of chunks, pinned or pageable host memory, with or without LSE.  It is also
checked against the float64 oracle directly on a small problem.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import make_qkv, sample_rows
from oracle import attention_rows

pytestmark = pytest.mark.gpu

FA_ERR_UNSUPPORTED = 3


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def device_reference(q, k, v, causal):
    from exact_softmax_attention_02_b200 import fa

    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:3], device="cuda")
    fa.fa_fwd(qd, kd, vd, o, lse, causal=causal)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def host_run(q, k, v, causal, chunks, pinned=True, with_lse=True):
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d = q.shape
    if pinned:
        q, k, v = (t.pin_memory() for t in (q, k, v))
    o = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, pin_memory=pinned)
    lse = torch.full((B, H, N), float("nan"), pin_memory=pinned) if with_lse else None
    ws = torch.empty(fa.host_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    fa.fa_fwd_host(q, k, v, o, lse, workspace=ws, chunks=chunks, causal=causal, stream=stream)
    stream.synchronize()
    assert fa.device_status_word() == 0
    return o, lse


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 1, 1, 64, False), (2, 3, 300, 128, True), (1, 5, 1000, 64, False),
                                            (2, 16, 2048, 128, True)])
@pytest.mark.parametrize("chunks", [0, 1, 3, 64])
def test_host_path_equals_device_path_bit_for_bit(B, H, N, d, causal, chunks):
    q, k, v = make_qkv(B, H, N, d, seed=B * 1000 + H * 10 + N)
    o_ref, lse_ref = device_reference(q, k, v, causal)
    o, lse = host_run(q, k, v, causal, chunks)
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_pageable_memory_and_no_lse():
    q, k, v = make_qkv(1, 4, 777, 128, seed=3)
    o_ref, _ = device_reference(q, k, v, True)
    o, lse = host_run(q, k, v, True, 2, pinned=False, with_lse=False)
    assert lse is None and torch.equal(o, o_ref)


def test_host_path_against_oracle():
    B, H, N, d = 1, 2, 640, 64
    q, k, v = make_qkv(B, H, N, d, seed=21)
    o, lse = host_run(q, k, v, False, 2)
    rows = sample_rows(B, H, N, 0, 0).numpy()
    ro, rl = attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), 1 / math.sqrt(d), False, rows)
    go = o.double().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    gl = lse.double().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert np.abs(go - ro).max() <= 2e-2 and np.abs(go - ro).mean() <= 2e-3 and np.abs(gl - rl).max() <= 1e-3


def test_back_to_back_calls_reuse_the_workspace():
    """Two calls on one workspace, the second issued before the first has finished."""
    from exact_softmax_attention_02_b200 import fa

    B, H, N, d = 1, 8, 2048, 128
    a = [t.pin_memory() for t in make_qkv(B, H, N, d, seed=31)]
    b = [t.pin_memory() for t in make_qkv(B, H, N, d, seed=32)]
    ws = torch.empty(fa.host_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    oa = torch.empty(a[0].shape, dtype=torch.bfloat16, pin_memory=True)
    ob = torch.empty(a[0].shape, dtype=torch.bfloat16, pin_memory=True)
    stream = torch.cuda.current_stream()
    fa.fa_fwd_host(*a, oa, None, workspace=ws, causal=True, stream=stream)
    fa.fa_fwd_host(*b, ob, None, workspace=ws, causal=True, stream=stream)
    stream.synchronize()
    assert torch.equal(oa, device_reference(*a, True)[0])
    assert torch.equal(ob, device_reference(*b, True)[0])


def test_device_memory_as_host_argument_is_refused():
    from exact_softmax_attention_02_b200 import fa

    lib = fa._load()
    B, H, N, d = 1, 1, 128, 64
    qd = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(fa.host_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
    host = torch.zeros((B, H, N, d), dtype=torch.bfloat16)
    st = lib.fa_fwd_host(qd.data_ptr(), host.data_ptr(), host.data_ptr(), host.data_ptr(), None,
                         ws.data_ptr(), ws.numel(), B, H, N, d, ctypes.c_float(0.125), 0, 0, None)
    assert st == FA_ERR_UNSUPPORTED
    # a host buffer passed as the workspace
    big = torch.empty(fa.host_workspace_bytes(B, H, N, d), dtype=torch.uint8)
    st = lib.fa_fwd_host(host.data_ptr(), host.data_ptr(), host.data_ptr(), host.data_ptr(), None,
                         big.data_ptr(), big.numel(), B, H, N, d, ctypes.c_float(0.125), 0, 0, None)
    assert st == FA_ERR_UNSUPPORTED


def test_attention_forward_on_host_tensors_uses_the_pipeline():
    from exact_softmax_attention_02_b200 import fa

    q, k, v = make_qkv(2, 4, 512, 64, seed=41)
    o, lse = fa.attention_forward(q, k, v, causal=True)
    o_ref, lse_ref = device_reference(q, k, v, True)
    assert not o.is_cuda and torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
