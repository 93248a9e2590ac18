"""ctypes binding of libfa.so (include/fa.h): argument marshalling only.

Every step of the attention forward runs in the library's CUDA kernel; this
module checks tensor properties, passes raw pointers and the current CUDA
stream, and turns status codes into exceptions.  There is no fallback: if the
library is missing or the device is not an sm_100 GPU, calls raise.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libfa.so"

FA_OK = 0
FA_ERR_DEVICE_TIMEOUT = 6
FA_ERR_LAYOUT = 9

# block of the block-sparse layout: query rows x keys (FA_BLOCK_Q, FA_BLOCK_K)
BLOCK_Q = 256
BLOCK_K = 128


class FAError(RuntimeError):
    """A libfa call returned a non-OK status."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def library_path() -> str:
    return os.environ.get("FA_LIBRARY", os.path.join(_HERE, _LIB_NAME))


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    _lib = load_library(library_path())
    return _lib


def load_library(path: str):
    """Open a build of libfa.so at ``path`` and declare its signatures.

    ``_load`` uses this for the library the module calls; the debug-build tests
    use it to open ``libfa_debug.so`` beside it."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} not found: build the CUDA library first "
            "(python -m exact_softmax_attention_02_b200.build)")
    lib = ctypes.CDLL(path)
    vp, c_int, c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_float, c_int, vp]
    lib.fa_fwd.restype = c_int
    lib.fa_status_string.argtypes = [c_int]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_get_device_status.argtypes = [vp]
    lib.fa_get_device_status.restype = c_int
    lib.fa_get_device_status_word.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    lib.fa_get_device_status_word.restype = c_int
    lib.fa_last_cuda_error.argtypes = []
    lib.fa_last_cuda_error.restype = ctypes.c_char_p
    lib.fa_set_debug.argtypes = [ctypes.c_uint, ctypes.c_ulonglong]
    lib.fa_set_debug.restype = None
    lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_size_t, c_int, c_int, c_int,
                                   c_int, c_float, c_int, c_int, vp]
    lib.fa_fwd_splitkv.restype = c_int
    lib.fa_fwd_splitkv_workspace_bytes.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int]
    lib.fa_fwd_splitkv_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_splitkv_default_splits.argtypes = [c_int, c_int, c_int, c_int, c_int]
    lib.fa_fwd_splitkv_default_splits.restype = c_int
    lib.fa_bwd.argtypes = [vp] * 10 + [ctypes.c_size_t, c_int, c_int, c_int, c_int, c_float, c_int, vp]
    lib.fa_bwd.restype = c_int
    lib.fa_bwd_workspace_bytes.argtypes = [c_int, c_int, c_int]
    lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_block_sparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int,
                                        c_float, c_int, vp]
    lib.fa_fwd_block_sparse.restype = c_int
    lib.fa_fwd_tile_config.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_float, c_int, c_int,
                                       c_int, vp]
    lib.fa_fwd_tile_config.restype = c_int
    lib.fa_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_size_t, c_int, c_int, c_int, c_int, c_float,
                                c_int, c_int, vp]
    lib.fa_fwd_host.restype = c_int
    lib.fa_fwd_host_workspace_bytes.argtypes = [c_int, c_int, c_int, c_int]
    lib.fa_fwd_host_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_version.argtypes = []
    lib.fa_version.restype = ctypes.c_char_p
    return lib


def _check(status: int):
    if status != FA_OK:
        lib = _load()
        msg = lib.fa_status_string(status).decode()
        detail = lib.fa_last_cuda_error().decode()
        raise FAError(status, f"{msg}{' (' + detail + ')' if detail else ''}")


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check_qkvo(q, k, v, o):
    shape = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.shape != shape:
            break
    if len(shape) != 4:
        raise ValueError("q must be [B, H, N, d]")
    if not (shape == k.shape == v.shape == o.shape):
        raise ValueError(f"shape mismatch: q{tuple(q.shape)} k{tuple(k.shape)} "
                         f"v{tuple(v.shape)} o{tuple(o.shape)}")


def _lse_ptr(lse, B: int, H: int, N: int):
    """Pointer of an optional fp32 [B, H, N] CUDA tensor (None -> NULL)."""
    if lse is None:
        return None
    if lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous CUDA float32 tensor")
    if tuple(lse.shape) != (B, H, N):
        raise ValueError(f"lse must be [B, H, N] = {(B, H, N)}")
    return lse.data_ptr()


def _launch_device_index(stream, first, *rest) -> int:
    """Index of the one CUDA device all tensors (and the stream) live on.

    The same check as _launch_device, on device indices: the cheaper form
    for the per-call path of fa_fwd."""
    dev = first.get_device()
    for t in rest:
        if t is not None and t.get_device() != dev:
            raise ValueError("all tensors must be on one CUDA device")
    if stream is not None and stream.device_index != dev:
        raise ValueError(f"stream is on cuda:{stream.device_index}, tensors on cuda:{dev}")
    return dev


def _launch_device(stream, *tensors) -> torch.device:
    """The one CUDA device every tensor (and the stream, if given) lives on.

    The kernels run on the current device and dereference every pointer there,
    so tensors spread over several devices are refused here."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all tensors must be on one CUDA device, got {sorted(str(d) for d in devs)}")
    dev = devs.pop()
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, tensors on {dev}")
    return dev


def fa_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
           lse: torch.Tensor | None = None, scale: float | None = None,
           causal: bool = False, stream=None) -> None:
    """Launch the fused forward: o = softmax(scale q k^T [causal]) v, lse.

    q, k, v, o: CUDA bfloat16 [B, H, N, d], contiguous (d = 64 or 128), on one
    device.  lse: CUDA float32 [B, H, N] contiguous, or None.
    scale: defaults to 1/sqrt(d).  Asynchronous on ``stream`` (default: the
    current stream of the tensors' device).
    """
    lib = _lib if _lib is not None else _load()
    _check_qkvo(q, k, v, o)
    B, H, N, d = q.shape
    lse_ptr = _lse_ptr(lse, B, H, N)
    dev = _launch_device_index(stream, q, k, v, o, lse)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    handle = stream.cuda_stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_ptr, B, H, N, d, float(scale),
            int(bool(causal)), handle)
    if torch.cuda.current_device() == dev:
        _check(lib.fa_fwd(*args))
    else:
        with torch.cuda.device(dev):
            _check(lib.fa_fwd(*args))


def fa_fwd_tile_config(q, k, v, o, lse=None, query_rows: int = 256, key_tile: int = 128,
                       scale: float | None = None, causal: bool = False, stream=None) -> None:
    """fa_fwd with ``query_rows`` (256 or 128) query rows per CTA and ``key_tile``
    (128 or 64) keys per score tile, for the tile-size sweep."""
    lib = _load()
    _check_qkvo(q, k, v, o)
    B, H, N, d = q.shape
    lse_ptr = _lse_ptr(lse, B, H, N)
    dev = _launch_device(stream, q, k, v, o, lse)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        _check(lib.fa_fwd_tile_config(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_ptr,
                                      B, H, N, d, float(scale), int(bool(causal)), int(query_rows),
                                      int(key_tile), _stream_handle(stream)))


def splitkv_workspace_bytes(B: int, H: int, N: int, d: int, num_splits: int = 0,
                            causal: bool = False) -> int:
    """Workspace bytes fa_fwd_splitkv needs (num_splits <= 0: the default)."""
    return int(_load().fa_fwd_splitkv_workspace_bytes(B, H, N, d, int(bool(causal)), num_splits))


def splitkv_default_splits(B: int, H: int, N: int, d: int, causal: bool = False) -> int:
    return int(_load().fa_fwd_splitkv_default_splits(B, H, N, d, int(bool(causal))))


def fa_fwd_splitkv(q, k, v, o, lse=None, workspace=None, num_splits: int = 0,
                   scale: float | None = None, causal: bool = False, stream=None) -> None:
    """Split-KV forward (same result as fa_fwd).  ``workspace``: a CUDA tensor
    of at least splitkv_workspace_bytes(...) bytes (allocated here if None)."""
    lib = _load()
    _check_qkvo(q, k, v, o)
    B, H, N, d = q.shape
    lse_ptr = _lse_ptr(lse, B, H, N)
    if workspace is None:
        nbytes = splitkv_workspace_bytes(B, H, N, d, num_splits, causal)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    dev = _launch_device(stream, q, k, v, o, lse, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        _check(lib.fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_ptr,
                                  workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                  B, H, N, d, float(scale), int(bool(causal)), int(num_splits),
                                  _stream_handle(stream)))


def block_layout_to_csr(layout, device=None):
    """CSR lists (row_ptr, col_idx), int32 on ``device``, of a boolean block layout.

    layout[r][c] set = query block r (rows BLOCK_Q*r ...) retains key block c
    (keys BLOCK_K*c ...); shape [ceil(N / BLOCK_Q), ceil(N / BLOCK_K)].
    Column indices come out ascending within each row, as fa_fwd_block_sparse
    requires.
    """
    lay = torch.as_tensor(layout, dtype=torch.bool, device=device)
    if lay.dim() != 2:
        raise ValueError("layout must be 2-D [query blocks, key blocks]")
    counts = lay.sum(dim=1, dtype=torch.int32)
    row_ptr = torch.zeros(lay.shape[0] + 1, dtype=torch.int32, device=lay.device)
    row_ptr[1:] = torch.cumsum(counts, 0)
    col_idx = lay.nonzero()[:, 1].to(torch.int32).contiguous()
    return row_ptr, col_idx


def fa_fwd_block_sparse(q, k, v, o, row_ptr, col_idx, lse=None, scale: float | None = None,
                        causal: bool = False, stream=None) -> None:
    """Block-sparse forward: attention over the key blocks each query block retains.

    row_ptr, col_idx: CUDA int32 CSR lists (see block_layout_to_csr), one
    layout for every (b, h).  Other arguments as fa_fwd.
    """
    lib = _load()
    _check_qkvo(q, k, v, o)
    B, H, N, d = q.shape
    n_qb = -(-N // BLOCK_Q)
    for name, t in (("row_ptr", row_ptr), ("col_idx", col_idx)):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.dim() != 1:
            raise ValueError(f"{name} must be a contiguous 1-D CUDA int32 tensor")
    if row_ptr.numel() != n_qb + 1:
        raise ValueError(f"row_ptr must have ceil(N / {BLOCK_Q}) + 1 = {n_qb + 1} entries")
    lse_ptr = _lse_ptr(lse, B, H, N)
    dev = _launch_device(stream, q, k, v, o, lse, row_ptr, col_idx)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nnz = col_idx.numel()
    with torch.cuda.device(dev):
        _check(lib.fa_fwd_block_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_ptr,
                                       row_ptr.data_ptr(), col_idx.data_ptr() if nnz else None, nnz,
                                       B, H, N, d, float(scale), int(bool(causal)),
                                       _stream_handle(stream)))


def bwd_workspace_bytes(B: int, H: int, N: int) -> int:
    """Workspace bytes fa_bwd needs."""
    return int(_load().fa_bwd_workspace_bytes(B, H, N))


def fa_bwd(q, k, v, o, do, lse, dq, dk, dv, workspace=None, scale: float | None = None,
           causal: bool = False, stream=None) -> None:
    """Backward pass: dq, dk, dv of L = sum(o * do) for o = fa_fwd(q, k, v).

    q, k, v, o, do, dq, dk, dv: CUDA bf16 [B, H, N, d] contiguous; lse: the
    forward's fp32 [B, H, N].  ``workspace``: at least
    fa_bwd_workspace_bytes(B, H, N) bytes of CUDA memory (allocated here if None).
    """
    lib = _load()
    _check_qkvo(q, k, v, o)
    _check_qkvo(do, dq, dk, dv)
    if do.shape != q.shape:
        raise ValueError("do, dq, dk, dv must have the shape of q")
    B, H, N, d = q.shape
    if lse is None:
        raise ValueError("lse (the forward's) is required")
    lse_ptr = _lse_ptr(lse, B, H, N)
    need = int(lib.fa_bwd_workspace_bytes(B, H, N))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    dev = _launch_device(stream, q, k, v, o, do, lse, dq, dk, dv, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        _check(lib.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                          lse_ptr, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          B, H, N, d, float(scale), int(bool(causal)), _stream_handle(stream)))


def host_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    """Device workspace bytes fa_fwd_host needs."""
    return int(_load().fa_fwd_host_workspace_bytes(B, H, N, d))


def fa_fwd_host(q, k, v, o, lse=None, workspace=None, chunks: int = 0, scale: float | None = None,
                causal: bool = False, stream=None) -> None:
    """The forward on HOST tensors, copies pipelined with the kernels (fa_fwd_host).

    q, k, v, o: CPU bf16 [B, H, N, d] contiguous (pinned for overlapping
    copies); lse: CPU float32 [B, H, N] or None.  ``workspace``: a CUDA
    tensor of at least host_workspace_bytes(...) bytes on the device to run
    on.  Asynchronous on ``stream``: synchronise it before reading o and lse.
    """
    lib = _load()
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous CPU bfloat16 [B, H, N, d] tensor")
    if not (q.shape == k.shape == v.shape == o.shape):
        raise ValueError("q, k, v, o must have the same shape")
    B, H, N, d = q.shape
    lse_ptr = None
    if lse is not None:
        if lse.dtype != torch.float32 or lse.is_cuda or not lse.is_contiguous() or tuple(lse.shape) != (B, H, N):
            raise ValueError(f"lse must be a contiguous CPU float32 [B, H, N] = {(B, H, N)} tensor")
        lse_ptr = lse.data_ptr()
    if workspace is None or not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    dev = _launch_device(stream, workspace)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        _check(lib.fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse_ptr,
                               workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                               B, H, N, d, float(scale), int(bool(causal)), int(chunks),
                               _stream_handle(stream)))


_host_workspaces = {}


def _host_workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    """A device workspace of at least ``nbytes``, kept per device for reuse."""
    ws = _host_workspaces.get(device)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        _host_workspaces[device] = ws
    return ws


def attention_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      scale: float | None = None, causal: bool = False,
                      return_lse: bool = True, device=None, out=None, num_splits=None):
    """Allocate the outputs and run the forward.

    CUDA inputs: outputs stay on their device.  CPU inputs (ideally pinned):
    fa_fwd_host copies them to ``device`` (default: the current CUDA device)
    and O (and LSE) back to host memory, pipelined with the kernels over
    groups of heads -- into ``out = (o_host, lse_host)`` when given (pinned
    buffers of the right shape and dtype, reused across calls), else into new
    pinned tensors.  The call returns after the copies have completed.
    ``num_splits`` (not None) runs the split-KV forward with that many key
    ranges (0: its default), with whole-tensor copies.
    """
    on_host = not q.is_cuda
    if on_host and num_splits is None:
        dev = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        if out is not None:
            o_h, lse_h = out
            if tuple(o_h.shape) != tuple(q.shape) or o_h.dtype != q.dtype:
                raise ValueError("out[0] must match q in shape and dtype")
            if return_lse and (lse_h is None or tuple(lse_h.shape) != tuple(q.shape[:3])):
                raise ValueError("out[1] must be a float32 [B, H, N] tensor")
        else:
            o_h = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
            lse_h = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True) if return_lse else None
        B, H, N, d = q.shape
        with torch.cuda.device(dev):
            ws = _host_workspace(dev, host_workspace_bytes(B, H, N, d))
            stream = torch.cuda.current_stream(dev)
            fa_fwd_host(q.contiguous(), k.contiguous(), v.contiguous(), o_h, lse_h if return_lse else None,
                        workspace=ws, scale=scale, causal=causal, stream=stream)
            stream.synchronize()
        return (o_h, lse_h) if return_lse else o_h
    if on_host:
        dev = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        q = q.to(dev, non_blocking=True)
        k = k.to(dev, non_blocking=True)
        v = v.to(dev, non_blocking=True)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) if return_lse else None
    if num_splits is None:
        fa_fwd(q, k, v, o, lse, scale=scale, causal=causal)
    else:
        fa_fwd_splitkv(q, k, v, o, lse, num_splits=num_splits, scale=scale, causal=causal)
    if not on_host:
        return (o, lse) if return_lse else o
    if out is not None:
        o_h, lse_h = out
        if tuple(o_h.shape) != tuple(o.shape) or o_h.dtype != o.dtype:
            raise ValueError("out[0] must match O in shape and dtype")
        if return_lse and (lse_h is None or tuple(lse_h.shape) != tuple(lse.shape)):
            raise ValueError("out[1] must be a float32 [B, H, N] tensor")
    else:
        o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True) if return_lse else None
    o_h.copy_(o, non_blocking=True)
    if return_lse:
        lse_h.copy_(lse, non_blocking=True)
    torch.cuda.current_stream(o.device).synchronize()
    return (o_h, lse_h) if return_lse else o_h


def device_status(stream=None) -> int:
    """Synchronise the stream and read-and-clear the library's device status."""
    return _load().fa_get_device_status(_stream_handle(stream))


def device_status_word(stream=None) -> int:
    """Synchronise, read and clear the raw device status word (0 = no failure;
    bit 0 = a bounded wait gave up, bit 8+k = the wait at site k gave up)."""
    w = ctypes.c_uint(0)
    _load().fa_get_device_status_word(_stream_handle(stream), ctypes.byref(w))
    return int(w.value)


def set_debug(flags: int = 0, timeout_ns: int = 0) -> None:
    """Test hook of include/fa.h (fa_set_debug)."""
    _load().fa_set_debug(int(flags), int(timeout_ns))


def version() -> str:
    return _load().fa_version().decode()
