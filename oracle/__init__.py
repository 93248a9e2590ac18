"""Float64 CPU oracle for exact softmax attention -- test infrastructure only.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its Python binding) never does, and this package imports nothing from
the product.
"""

from .attention import (  # noqa: F401
    attention_backward,
    attention_full,
    attention_rows,
    block_layout_from_csr,
    block_sparse_attention_rows,
    brute_force_attention,
    flops_for_rows,
    merge_block,
    merge_states,
    online_attention_rows,
    scalar_online_weighted_sum,
    scalar_softmax_weighted_sum,
)
