"""Standard (materialising) attention on the GPU, the comparator of the fused path.

It computes the same O = softmax(scale * Q K^T [+ causal mask]) V the way a
conventional implementation does.  It writes the N x N scores to global
memory, reads them back for the softmax, writes the probabilities, and reads
them again for the product with V (sadullah.online "Flash Attention
Explained", the memory-movement section; lihaoran.work, the N x N
intermediate matrix).  The pages set the fused kernel against exactly this:
"2-4x faster" (sadullah.online, comparison table) and "up to 9x fewer HBM
accesses" (interactiveml.org).

Steps per group of heads:
  1. S = Q K^T  -- cuBLAS GEMM, bf16 inputs, fp32 accumulate and output.
  2. P = softmax(scale * S), LSE -- this library's fa_softmax_rows kernel.
  3. O = P V    -- cuBLAS GEMM, bf16 inputs and output, fp32 accumulate.
The GEMMs are plain library GEMMs, called through the cuBLAS that PyTorch
loads.  S (fp32) and P (bf16) are allocated per head group, within a memory
budget.
"""

from __future__ import annotations

import ctypes
import glob
import math
import os

import torch

from . import fa

_CUBLAS_OP_N, _CUBLAS_OP_T = 0, 1
_CUDA_R_32F, _CUDA_R_16BF = 0, 14
_CUBLAS_COMPUTE_32F = 68
_CUBLAS_GEMM_DEFAULT = -1

_cublas = None
_handles = {}


def _load_cublas():
    global _cublas
    if _cublas is not None:
        return _cublas
    cands = []
    try:
        import nvidia.cublas

        for d in nvidia.cublas.__path__:
            cands += glob.glob(os.path.join(d, "lib", "libcublas.so*"))
    except ImportError:
        pass
    cands.append("libcublas.so.12")
    last = None
    for c in cands:
        try:
            lib = ctypes.CDLL(c)
            break
        except OSError as e:
            last = e
    else:
        raise RuntimeError(f"cuBLAS not found: {last}")
    vp, ci, cll = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    lib.cublasCreate_v2.argtypes = [ctypes.POINTER(vp)]
    lib.cublasCreate_v2.restype = ci
    lib.cublasSetStream_v2.argtypes = [vp, vp]
    lib.cublasSetStream_v2.restype = ci
    lib.cublasGemmStridedBatchedEx.argtypes = [
        vp, ci, ci, ci, ci, ci, vp, vp, ci, ci, cll, vp, ci, ci, cll, vp, vp, ci, ci, cll, ci, ci, ci]
    lib.cublasGemmStridedBatchedEx.restype = ci
    _cublas = lib
    return lib


def _handle(device: torch.device):
    idx = device.index if device.index is not None else torch.cuda.current_device()
    if idx not in _handles:
        lib = _load_cublas()
        h = ctypes.c_void_p()
        with torch.cuda.device(idx):
            st = lib.cublasCreate_v2(ctypes.byref(h))
        if st != 0:
            raise RuntimeError(f"cublasCreate failed: {st}")
        _handles[idx] = h
    return _handles[idx]


def _gemm(h, ta, tb, m, n, k, A, lda, sa, B, ldb, sb, C, ctype, ldc, sc, batch):
    lib = _load_cublas()
    one = ctypes.c_float(1.0)
    zero = ctypes.c_float(0.0)
    st = lib.cublasGemmStridedBatchedEx(
        h, ta, tb, m, n, k, ctypes.byref(one), A, _CUDA_R_16BF, lda, sa, B, _CUDA_R_16BF, ldb, sb,
        ctypes.byref(zero), C, ctype, ldc, sc, batch, _CUBLAS_COMPUTE_32F, _CUBLAS_GEMM_DEFAULT)
    if st != 0:
        raise RuntimeError(f"cublasGemmStridedBatchedEx failed: {st}")


def heads_per_group(N: int, budget_bytes: int = 48 << 30) -> int:
    """How many heads' S (fp32) and P (bf16) fit in the budget at once."""
    return max(1, budget_bytes // (6 * N * N))


def standard_attention(q, k, v, o=None, lse=None, scale: float | None = None, causal: bool = False,
                       budget_bytes: int = 48 << 30, buffers=None, softmax_events=None):
    """O = softmax(scale q k^T [causal]) v with the N x N matrices in memory.

    q, k, v: CUDA bf16 [B, H, N, d] contiguous.  Returns (o, lse).  ``buffers``
    may pass preallocated (S fp32, P bf16) tensors of at least one head
    group; otherwise they are allocated here.  ``softmax_events``, a list,
    receives a (start, end) pair of CUDA events around each softmax launch.
    Asynchronous on the current stream.
    """
    fa._check_qkvo(q, k, v, q if o is None else o)
    B, H, N, d = q.shape
    if N % 2:
        raise ValueError("the comparator's softmax needs an even N")
    BH = B * H
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    g = min(BH, heads_per_group(N, budget_bytes))
    if buffers is None:
        S = torch.empty((g, N, N), dtype=torch.float32, device=q.device)
        P = torch.empty((g, N, N), dtype=torch.bfloat16, device=q.device)
    else:
        S, P = buffers
    h = _handle(q.device)
    stream = torch.cuda.current_stream(q.device)
    _load_cublas().cublasSetStream_v2(h, ctypes.c_void_p(stream.cuda_stream))
    lib = fa._load()
    lib.fa_softmax_rows.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    lib.fa_softmax_rows.restype = ctypes.c_int
    qf, kf, vf, of = (t.view(BH, N, d) for t in (q, k, v, o))
    lf = lse.view(BH, N)
    for h0 in range(0, BH, g):
        n = min(g, BH - h0)
        # S^T (column-major) = K Q^T, i.e. row-major S[i][j] = q_i . k_j
        _gemm(h, _CUBLAS_OP_T, _CUBLAS_OP_N, N, N, d, kf[h0].data_ptr(), d, N * d,
              qf[h0].data_ptr(), d, N * d, S.data_ptr(), _CUDA_R_32F, N, N * N, n)
        if softmax_events is not None:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(stream)
        fa._check(lib.fa_softmax_rows(S.data_ptr(), P.data_ptr(), lf[h0].data_ptr(), n, N,
                                      float(scale), int(bool(causal)), stream.cuda_stream))
        if softmax_events is not None:
            ev[1].record(stream)
            softmax_events.append(ev)
        # O^T (column-major) = V^T P^T, i.e. row-major O = P V
        _gemm(h, _CUBLAS_OP_N, _CUBLAS_OP_N, d, N, N, vf[h0].data_ptr(), d, N * d,
              P.data_ptr(), N, N * N, of[h0].data_ptr(), _CUDA_R_16BF, d, N * d, n)
    return o, lse
