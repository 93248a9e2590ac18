"""The no-allocation split-KV entry point, called through the C ABI.

Some callers cannot allocate device memory when they run attention -- code
being captured into a CUDA graph, runtimes that forbid allocation after
start-up, programs whose memory belongs to another framework's pool -- so
fa_fwd_splitkv_noalloc runs the split-KV forward on a 64 MiB array built into
the library instead of a caller's workspace.  These tests check that

- it gives bit for bit the result of fa_fwd_splitkv with a caller workspace
  (the same kernels on the same inputs), on a shape called twice in a row
  right after a different shape, so that whatever an earlier call left in the
  shared array is really there when the next call runs;
- that result also matches the float64 oracle on every row, within the
  tolerances of the other parity tests;
- a problem that runs as a single key range needs no scratch and is served
  whatever its size, and a problem whose partial states exceed the array is
  refused before anything runs.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import make_qkv
from oracle import attention_rows

pytestmark = pytest.mark.gpu

FA_OK, FA_ERR_WORKSPACE = 0, 8
O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_softmax_attention_02_b200 import fa

    handle = fa._load()
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    handle.fa_fwd_splitkv_noalloc.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, ci, ci, vp]
    handle.fa_fwd_splitkv_noalloc.restype = ci
    return handle


def _noalloc(lib, q, k, v, causal, num_splits):
    B, H, N, d = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device=q.device)
    stream = torch.cuda.current_stream().cuda_stream
    status = lib.fa_fwd_splitkv_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), B, H, N, d, 1.0 / math.sqrt(d),
                                        int(causal), num_splits, stream)
    return status, o, lse


def _with_workspace(q, k, v, causal, num_splits):
    from exact_softmax_attention_02_b200 import fa

    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], device=q.device)
    fa.fa_fwd_splitkv(q, k, v, o, lse, num_splits=num_splits, causal=causal)
    return o, lse


def _check_oracle(q, k, v, causal, o, lse):
    B, H, N, d = q.shape
    rows = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(N)])
    ro, rl = attention_rows(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(),
                            1.0 / math.sqrt(d), causal, rows)
    go = o.cpu().double().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    gl = lse.cpu().double().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    err, lerr = np.abs(go - ro), np.abs(gl - rl)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN and lerr.max() <= LSE_MAX, \
        (err.max(), err.mean(), lerr.max())


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    from exact_softmax_attention_02_b200 import fa

    # (shape, causal, requested ranges, seed): the first case fills the array
    # with partial states of another shape, then the second runs twice
    first = ((1, 1, 4096, 64), False, 0, 42)
    second = ((1, 2, 1000, 128), True, 3, 41)
    for (B, H, N, d), causal, splits, seed in (first, second, second):
        q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=seed))
        status, o, lse = _noalloc(lib, q, k, v, causal, splits)
        assert status == FA_OK, lib.fa_status_string(status)
        assert fa.device_status_word() == 0
        o_ref, lse_ref = _with_workspace(q, k, v, causal, splits)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, lse_ref)
        _check_oracle(q, k, v, causal, o, lse)


def test_noalloc_single_range_needs_no_scratch(lib):
    from exact_softmax_attention_02_b200 import fa

    # one key range: the fused kernel writes O and LSE directly, so even a
    # problem whose ranges would not fit in the array runs
    B, H, N, d = 2, 16, 8192, 128
    q, k, v = (torch.randn((B, H, N, d), device="cuda").to(torch.bfloat16) for _ in range(3))
    status, o, lse = _noalloc(lib, q, k, v, True, 1)
    assert status == FA_OK, lib.fa_status_string(status)
    assert fa.device_status_word() == 0
    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, N), device="cuda")
    fa.fa_fwd(q, k, v, o_ref, lse_ref, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)


def test_noalloc_refuses_a_problem_larger_than_its_array(lib):
    # 8 heads x 32768 rows x (128 + 1) floats x 2 ranges = 270 MB > 64 MiB
    B, H, N, d = 1, 8, 32768, 128
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    status, _, _ = _noalloc(lib, q, q, q, False, 2)
    assert status == FA_ERR_WORKSPACE
