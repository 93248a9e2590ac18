"""The no-allocation split-KV entry point, called through the C ABI.

Some callers cannot allocate device memory when they run attention -- code
being captured into a CUDA graph, runtimes that forbid allocation after
start-up, programs whose memory belongs to another framework's pool -- so
fa_fwd_splitkv_noalloc runs the split-KV forward on a 64 MiB array built into
the library instead of a caller's workspace.  These tests check that it gives
the same result as fa_fwd_splitkv with a caller workspace, on two calls in a
row (the array keeps the previous call's contents), and that a problem too
large for the array is refused before anything runs.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes
import math

import pytest
import torch

from exact_softmax_attention_02_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

FA_OK, FA_ERR_WORKSPACE = 0, 8
O_TOL, LSE_TOL = 2e-2, 1e-3


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


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    from exact_softmax_attention_02_b200 import fa

    cases = [((1, 2, 1000, 128), True, 3, 41), ((1, 1, 4096, 64), False, 0, 42)]
    for (B, H, N, d), causal, splits, seed in cases:
        q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=seed))
        status, o, lse = _noalloc(lib, q, k, v, causal, splits)
        assert status == FA_OK, lib.fa_status_string(status)
        assert fa.device_status_word() == 0
        o_ref, lse_ref = _with_workspace(q, k, v, causal, splits)
        torch.cuda.synchronize()
        assert not torch.isnan(o).any() and not torch.isnan(lse).any()
        assert (o.float() - o_ref.float()).abs().max().item() <= O_TOL
        assert (lse - lse_ref).abs().max().item() <= LSE_TOL


def test_noalloc_refuses_a_problem_larger_than_its_array(lib):
    # 8 heads x 32768 rows x (128 + 1) floats x 2 ranges = 270 MB > 64 MiB
    B, H, N, d = 1, 8, 32768, 128
    q = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    status, _, _ = _noalloc(lib, q, q, q, False, 2)
    assert status == FA_ERR_WORKSPACE
