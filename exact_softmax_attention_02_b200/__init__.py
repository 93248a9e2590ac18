"""Exact softmax attention for B200 (sm_100a): forward, split-KV, block-sparse,
host-buffer and backward paths.

The compute path is the C-ABI library ``libfa.so`` built from ``csrc/``;
``fa.py`` is its thin ctypes binding.  Importing this package does not load
the library; the first call does, and raises if it is missing.
"""

__all__ = [
    "fa_fwd", "fa_fwd_splitkv", "fa_fwd_block_sparse", "fa_fwd_tile_config", "fa_fwd_host", "fa_bwd",
    "attention_forward", "block_layout_to_csr", "device_status", "FAError", "library_path",
]


def __getattr__(name):
    if name in __all__:
        from . import fa

        return getattr(fa, name)
    raise AttributeError(name)
