"""CPU oracle for block-causal chunk attention over a bounded streaming KV cache.

TEST INFRASTRUCTURE.  This package is the plain, slow, fp64 statement of what
the hot path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import it.  The product path
(the C-ABI library ``libfd.so`` and its Python binding) never imports, links or
calls anything here, and the two share no code: no kernels, helpers, tables or
constants.  Inputs come from the seeded generators in
``streaming_autoregressive_video_b200.synth``, which hold none of the method's
arithmetic.

Every function pinned by ``tests/test_oracle.py`` against closed forms,
invariants and brute force; see the per-function docstrings for the passage
each one follows.  Parity unpinned: none.
"""
from .streaming_attention import (  # noqa: F401
    bf16_bits_to_f64,
    values_f64,
    rope_sections,
    rope_inv_freq,
    rope_angles,
    rope_rotate,
    token_coords,
    slot_of,
    valid_slot_count,
    RolloutCache,
    window_boundary_reached,
    start_window,
    block_attention,
    combine_partials,
)
