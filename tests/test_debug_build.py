"""The index-checking debug build, libfa_debug.so (-DFA_DEBUG).

In that build the forward and merge kernels check every shared-memory,
tensor-memory and global index they compute before using it; a failed check
sets a bit of the device status word and skips the access instead of
trapping.  On the CPU: the build compiles and exports the whole C ABI.  On
the GPU: small problems that exercise every mode of the forward kernel (fused,
split-KV with its merge, block-sparse, the other tile shapes, ragged tails,
both masks and head widths) run through it with no check failing, and give
the oracle's result within the usual tolerances.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from exact_softmax_attention_02_b200.inputs import make_qkv
from oracle import attention_rows, block_sparse_attention_rows

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module")
def debug_lib_path():
    from exact_softmax_attention_02_b200.build import build

    return build(debug=True)


def test_debug_build_exports_the_abi(debug_lib_path):
    from test_boundary import declared_functions

    lib = ctypes.CDLL(debug_lib_path)
    for name in declared_functions():
        assert hasattr(lib, name), f"libfa_debug.so does not export {name}"


@pytest.fixture()
def debug_fa(debug_lib_path, monkeypatch):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_softmax_attention_02_b200 import fa

    handle = fa.load_library(debug_lib_path)
    monkeypatch.setattr(fa, "_lib", handle)
    yield fa
    assert fa.device_status_word() == 0


def _rows(B, H, N):
    return np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(N)])


def _check(q, k, v, causal, o, lse, oracle=None):
    B, H, N, d = q.shape
    rows = _rows(B, H, N)
    if oracle is None:
        ro, rl = attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(), 1 / math.sqrt(d),
                                causal, rows)
    else:
        ro, rl = oracle(rows)
    go = o.cpu().double().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    gl = lse.cpu().double().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    err = np.abs(go - ro)
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(gl), fin)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN, (err.max(), err.mean())
    assert np.abs(gl[fin] - rl[fin]).max(initial=0.0) <= LSE_MAX


def _word(fa):
    word = fa.device_status_word()
    assert word == 0, f"device status word {word:#x}"


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 256, 300])
def test_fused_forward_passes_every_index_check(debug_fa, d, causal, N):
    fa = debug_fa
    q, k, v = make_qkv(1, 2, N, d, seed=N + d)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:3], float("nan"), device="cuda")
    fa.fa_fwd(qd, kd, vd, o, lse, causal=causal)
    _word(fa)
    _check(q, k, v, causal, o, lse)


@pytest.mark.gpu
@pytest.mark.parametrize("query_rows,key_tile", [(256, 64), (128, 128), (128, 64)])
def test_tile_shapes_pass_every_index_check(debug_fa, query_rows, key_tile):
    fa = debug_fa
    q, k, v = make_qkv(1, 2, 300, 128, seed=7)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:3], float("nan"), device="cuda")
    fa.fa_fwd_tile_config(qd, kd, vd, o, lse, causal=True, query_rows=query_rows, key_tile=key_tile)
    _word(fa)
    _check(q, k, v, True, o, lse)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_splitkv_and_merge_pass_every_index_check(debug_fa, causal):
    fa = debug_fa
    q, k, v = make_qkv(1, 2, 1000, 64, seed=3)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:3], float("nan"), device="cuda")
    fa.fa_fwd_splitkv(qd, kd, vd, o, lse, num_splits=3, causal=causal)
    _word(fa)
    _check(q, k, v, causal, o, lse)


@pytest.mark.gpu
def test_block_sparse_passes_every_index_check(debug_fa):
    fa = debug_fa
    N, d = 700, 128
    q, k, v = make_qkv(1, 2, N, d, seed=9)
    rng = np.random.default_rng(4)
    nqb, nkb = -(-N // fa.BLOCK_Q), -(-N // fa.BLOCK_K)
    layout = rng.random((nqb, nkb)) < 0.5
    layout[1, :] = False  # one query block with no retained key
    row_ptr, col_idx = fa.block_layout_to_csr(layout, device="cuda")
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:3], float("nan"), device="cuda")
    fa.fa_fwd_block_sparse(qd, kd, vd, o, row_ptr, col_idx, lse, causal=False)
    _word(fa)
    _check(q, k, v, False, o, lse,
           oracle=lambda rows: block_sparse_attention_rows(
               q.float().numpy(), k.float().numpy(), v.float().numpy(), 1 / math.sqrt(d), False, rows,
               layout, fa.BLOCK_Q, fa.BLOCK_K))
