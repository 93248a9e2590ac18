"""Exact softmax attention forward for B200 (sm_100a).

The compute path is the C-ABI library ``libfa.so`` built from ``csrc/``;
``fa.py`` is its thin ctypes binding.  Importing this package does not load
the library; the first call does, and raises if it is missing.
"""

__all__ = ["fa_fwd", "attention_forward", "FAError", "library_path"]


def __getattr__(name):
    if name in __all__:
        from . import fa

        return getattr(fa, name)
    raise AttributeError(name)
