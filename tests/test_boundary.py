"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and rejects bad arguments before anything is launched.

Only argument combinations that fail validation are passed (fake pointers
never reach a launch), so these tests are safe on any machine.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")
LIB = os.path.join(ROOT, "exact_softmax_attention_02_b200", "libfa.so")

FA_OK, FA_ERR_NULL, FA_ERR_SHAPE, FA_ERR_UNSUPPORTED, FA_ERR_ALIGN = 0, 1, 2, 3, 4
FA_ERR_CUDA, FA_ERR_DEVICE_TIMEOUT, FA_ERR_ALIAS, FA_ERR_WORKSPACE = 5, 6, 7, 8
FA_ERR_LAYOUT = 9


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from exact_softmax_attention_02_b200.build import build

        build()
    lib = ctypes.CDLL(LIB)
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, cf, ci, vp]
    lib.fa_fwd.restype = ci
    lib.fa_status_string.argtypes = [ci]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_version.restype = ctypes.c_char_p
    return lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa_fwd", "fa_status_string", "fa_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libfa.so does not export {name}"


def test_status_strings(lib):
    for code in range(11):
        s = lib.fa_status_string(code).decode()
        assert s.startswith("FA_")
    assert lib.fa_status_string(99).decode() == "unknown fa_status"
    assert re.match(r"^\d+\.\d+\.\d+$", lib.fa_version().decode())


A = 0x10000000  # fake, 16-byte-aligned "device" addresses: never dereferenced
MB = 1 << 20


def call(lib, q=A, k=A + 64 * MB, v=A + 128 * MB, o=A + 192 * MB, lse=A + 256 * MB,
         B=1, H=1, N=128, d=64, scale=0.125, causal=0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, None)


def test_null_pointers(lib):
    assert call(lib, q=None) == FA_ERR_NULL
    assert call(lib, k=None) == FA_ERR_NULL
    assert call(lib, v=None) == FA_ERR_NULL
    assert call(lib, o=None) == FA_ERR_NULL


@pytest.mark.parametrize("B,H,N", [(0, 1, 128), (1, 0, 128), (1, 1, 0), (-1, 1, 128), (1, 1, -5),
                                   (1 << 20, 1 << 20, 128)])
def test_bad_shapes(lib, B, H, N):
    assert call(lib, B=B, H=H, N=N) == FA_ERR_SHAPE


@pytest.mark.parametrize("d", [0, 32, 96, 256, 65])
def test_unsupported_head_width(lib, d):
    assert call(lib, d=d) == FA_ERR_UNSUPPORTED


def test_bad_scale(lib):
    assert call(lib, scale=float("nan")) == FA_ERR_SHAPE
    assert call(lib, scale=float("inf")) == FA_ERR_SHAPE
    assert call(lib, scale=0.0) == FA_ERR_UNSUPPORTED
    assert call(lib, scale=-0.5) == FA_ERR_UNSUPPORTED


def test_misaligned(lib):
    assert call(lib, q=A + 8) == FA_ERR_ALIGN
    assert call(lib, v=A + 128 * MB + 2) == FA_ERR_ALIGN
    assert call(lib, o=A + 192 * MB + 4) == FA_ERR_ALIGN
    assert call(lib, lse=A + 256 * MB + 2) == FA_ERR_ALIGN


def test_aliasing(lib):
    # O overlapping an input
    assert call(lib, o=A + 64) == FA_ERR_ALIAS
    # LSE inside O
    assert call(lib, lse=A + 192 * MB + 1024) == FA_ERR_ALIAS
    # LSE overlapping V
    assert call(lib, lse=A + 128 * MB) == FA_ERR_ALIAS


# split-KV entry point: workspace checks run before any device call
def _splitkv(lib, ws=A + 512 * MB, ws_bytes=1 << 30, num_splits=2, **kw):
    lib.fa_fwd_splitkv.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_size_t] + [ctypes.c_int] * 4 + \
        [ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    lib.fa_fwd_splitkv.restype = ctypes.c_int
    args = dict(q=A, k=A + 64 * MB, v=A + 128 * MB, o=A + 192 * MB, lse=A + 256 * MB,
                B=1, H=1, N=1024, d=64, scale=0.125, causal=0)
    args.update(kw)
    return lib.fa_fwd_splitkv(args["q"], args["k"], args["v"], args["o"], args["lse"], ws, ws_bytes,
                              args["B"], args["H"], args["N"], args["d"], args["scale"],
                              args["causal"], num_splits, None)


def test_splitkv_workspace_checks(lib):
    lib.fa_fwd_splitkv_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.fa_fwd_splitkv_workspace_bytes.restype = ctypes.c_size_t
    need = lib.fa_fwd_splitkv_workspace_bytes(1, 1, 1024, 64, 0, 2)
    assert need == 2 * 1024 * (64 + 1) * 4
    assert lib.fa_fwd_splitkv_workspace_bytes(1, 1, 1024, 96, 0, 2) == 0
    # the default split count depends on the mask
    assert lib.fa_fwd_splitkv_workspace_bytes(1, 2, 8192, 128, 1, 0) == 4 * 2 * 8192 * 129 * 4
    # sized for the ranges that remain: 100 requested over 8 key tiles runs 8
    assert lib.fa_fwd_splitkv_workspace_bytes(1, 1, 1024, 64, 0, 100) == 8 * 1024 * 65 * 4
    # a single range runs the fused kernel alone and needs no workspace
    assert lib.fa_fwd_splitkv_workspace_bytes(2, 16, 8192, 128, 1, 1) == 0
    assert lib.fa_fwd_splitkv_workspace_bytes(1, 1, 100, 64, 0, 4) == 0
    assert _splitkv(lib, ws=None) == FA_ERR_NULL
    assert _splitkv(lib, ws=A + 512 * MB + 4) == FA_ERR_ALIGN
    assert _splitkv(lib, ws_bytes=need - 4) == FA_ERR_WORKSPACE
    assert _splitkv(lib, num_splits=300) == FA_ERR_UNSUPPORTED
    assert _splitkv(lib, ws=A + 128 * MB + 1024) == FA_ERR_ALIAS  # inside V
    assert _splitkv(lib, q=None) == FA_ERR_NULL
    assert _splitkv(lib, d=32) == FA_ERR_UNSUPPORTED


def test_splitkv_default_splits(lib):
    lib.fa_fwd_splitkv_default_splits.argtypes = [ctypes.c_int] * 5
    lib.fa_fwd_splitkv_default_splits.restype = ctypes.c_int
    # 2 heads x 32 query blocks = 64 CTAs: one wave of 148 SMs (1.5 causal)
    assert lib.fa_fwd_splitkv_default_splits(1, 2, 8192, 128, 0) == 2
    assert lib.fa_fwd_splitkv_default_splits(1, 2, 8192, 128, 1) == 4
    assert lib.fa_fwd_splitkv_default_splits(1, 1, 32768, 128, 1) == 2
    # already many CTAs: no split
    assert lib.fa_fwd_splitkv_default_splits(4, 16, 4096, 64, 0) == 1
    # at least two key tiles per range
    assert lib.fa_fwd_splitkv_default_splits(1, 1, 512, 64, 0) == 2


def test_bwd_argument_checks(lib):
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_bwd.argtypes = [vp] * 10 + [ctypes.c_size_t, ci, ci, ci, ci, cf, ci, vp]
    lib.fa_bwd.restype = ci
    lib.fa_bwd_workspace_bytes.argtypes = [ci, ci, ci]
    lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    # LSE*log2(e) and D per padded row, then the fp32 dQ accumulator (d <= 128)
    assert lib.fa_bwd_workspace_bytes(2, 3, 100) == (2 + 128) * 2 * 3 * 128 * 4
    assert lib.fa_bwd_workspace_bytes(1, 1, 129) == (2 + 128) * 256 * 4
    base = [A + k * 64 * MB for k in range(10)]  # Q K V O dO LSE dQ dK dV ws

    def bwd(args=None, ws_bytes=1 << 20, N=128, d=64):
        a = list(base if args is None else args)
        return lib.fa_bwd(*a, ws_bytes, 1, 1, N, d, 0.125, 0, None)

    for idx in range(10):
        a = list(base)
        a[idx] = None
        assert bwd(a) == FA_ERR_NULL
    assert bwd(d=96) == FA_ERR_UNSUPPORTED
    assert bwd(N=0) == FA_ERR_SHAPE
    assert bwd(ws_bytes=2 * 128 * 4 - 4) == FA_ERR_WORKSPACE
    a = list(base)
    a[6] = base[0] + 32  # dQ overlapping Q
    assert bwd(a) == FA_ERR_ALIAS
    a = list(base)
    a[9] = base[6]  # workspace inside dQ
    assert bwd(a) == FA_ERR_ALIAS
    a = list(base)
    a[7] = base[7] + 8
    assert bwd(a) == FA_ERR_ALIGN


def test_block_sparse_argument_checks(lib):
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd_block_sparse.argtypes = [vp] * 7 + [ci] * 5 + [cf, ci, vp]
    lib.fa_fwd_block_sparse.restype = ci
    rp, ci_ = A + 320 * MB, A + 321 * MB

    def bs(q=A, o=A + 192 * MB, lse=A + 256 * MB, row_ptr=rp, col_idx=ci_, nnz=4, N=1024, d=64):
        return lib.fa_fwd_block_sparse(q, A + 64 * MB, A + 128 * MB, o, lse, row_ptr, col_idx, nnz,
                                       1, 1, N, d, 0.125, 0, None)

    assert bs(q=None) == FA_ERR_NULL
    assert bs(row_ptr=None) == FA_ERR_NULL
    assert bs(col_idx=None) == FA_ERR_NULL
    assert bs(nnz=-1) == FA_ERR_SHAPE
    assert bs(row_ptr=rp + 2) == FA_ERR_ALIGN
    assert bs(col_idx=ci_ + 1) == FA_ERR_ALIGN
    assert bs(d=96) == FA_ERR_UNSUPPORTED
    assert bs(row_ptr=A + 192 * MB + 64) == FA_ERR_ALIAS  # list inside O
    assert bs(col_idx=A + 256 * MB) == FA_ERR_ALIAS  # list inside LSE
    assert lib.fa_status_string(FA_ERR_LAYOUT).decode().startswith("FA_ERR_LAYOUT")


def test_tile_config_argument_checks(lib):
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd_tile_config.argtypes = [vp] * 5 + [ci] * 4 + [cf, ci, ci, ci, vp]
    lib.fa_fwd_tile_config.restype = ci

    def tc(query_rows, key_tile, q=A, d=64):
        return lib.fa_fwd_tile_config(q, A + 64 * MB, A + 128 * MB, A + 192 * MB, A + 256 * MB,
                                      1, 1, 1024, d, 0.125, 0, query_rows, key_tile, None)

    assert tc(256, 96) == FA_ERR_UNSUPPORTED
    assert tc(256, 256) == FA_ERR_UNSUPPORTED
    assert tc(64, 128) == FA_ERR_UNSUPPORTED
    assert tc(512, 64) == FA_ERR_UNSUPPORTED
    assert tc(128, 64, q=None) == FA_ERR_NULL
    assert tc(128, 128, d=32) == FA_ERR_UNSUPPORTED
    assert tc(0, 0, q=A + 8) == FA_ERR_ALIGN


def test_host_forward_argument_checks(lib):
    vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd_host.argtypes = [vp] * 6 + [ctypes.c_size_t] + [ci] * 4 + [cf, ci, ci, vp]
    lib.fa_fwd_host.restype = ci
    lib.fa_fwd_host_workspace_bytes.argtypes = [ci] * 4
    lib.fa_fwd_host_workspace_bytes.restype = ctypes.c_size_t
    need = lib.fa_fwd_host_workspace_bytes(2, 3, 100, 64)
    assert need == 4 * 2 * 3 * 100 * 64 * 2 + 2 * 3 * 100 * 4
    assert lib.fa_fwd_host_workspace_bytes(1, 1, 100, 96) == 0
    ws = A + 512 * MB

    def fh(q=A, ws=ws, ws_bytes=1 << 30, N=1024, d=64, scale=0.125):
        return lib.fa_fwd_host(q, A + 64 * MB, A + 128 * MB, A + 192 * MB, A + 256 * MB, ws, ws_bytes,
                               1, 1, N, d, scale, 0, 0, None)

    assert fh(q=None) == FA_ERR_NULL
    assert fh(ws=None) == FA_ERR_NULL
    assert fh(N=0) == FA_ERR_SHAPE
    assert fh(d=96) == FA_ERR_UNSUPPORTED
    assert fh(scale=-1.0) == FA_ERR_UNSUPPORTED
    assert fh(ws=ws + 8) == FA_ERR_ALIGN
    assert fh(ws_bytes=lib.fa_fwd_host_workspace_bytes(1, 1, 1024, 64) - 4) == FA_ERR_WORKSPACE
