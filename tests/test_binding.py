"""Argument checks of the Python binding that need no GPU."""

import pytest
import torch

from exact_softmax_attention_02_b200 import fa


def test_tensors_on_several_devices_are_refused():
    a = torch.zeros(4)
    b = torch.zeros(4, device="meta")
    with pytest.raises(ValueError, match="one CUDA device"):
        fa._launch_device(None, a, b)
    assert fa._launch_device(None, a, None, a) == a.device


def test_lse_checks():
    B, H, N = 2, 3, 5
    assert fa._lse_ptr(None, B, H, N) is None
    with pytest.raises(ValueError, match="contiguous CUDA float32"):
        fa._lse_ptr(torch.zeros(B, H, N), B, H, N)  # a CPU tensor


def test_qkvo_checks():
    q = torch.zeros(1, 1, 4, 64, dtype=torch.float32)
    with pytest.raises(TypeError):
        fa._check_qkvo(q, q, q, q)
    qb = q.to(torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        fa._check_qkvo(qb, qb, qb, qb)


def test_block_layout_to_csr_on_cpu():
    lay = [[True, False, True], [False, False, False], [False, True, True]]
    rp, ci = fa.block_layout_to_csr(lay)
    assert rp.tolist() == [0, 2, 2, 4] and ci.tolist() == [0, 2, 1, 2]
    assert rp.dtype == torch.int32 and ci.dtype == torch.int32


def test_host_forward_refuses_cuda_and_non_bf16_inputs():
    import os

    if not os.path.exists(fa.library_path()):
        from exact_softmax_attention_02_b200.build import build

        build()
    x = torch.zeros(1, 1, 8, 64, dtype=torch.float32)
    with pytest.raises(ValueError, match="CPU bfloat16"):
        fa.fa_fwd_host(x, x, x, x, workspace=None)
