"""CPU oracle (float64 NumPy) for the GSA layer and dense global attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package entry's
``smoke()`` check and by the benchmark's CPU-baseline / reference legs.  The
product path (the CUDA library and its Python binding) never imports it.

Parity status of every function here: pinned by the CPU tests in
``tests/test_oracle_pins.py`` (closed forms, library routines, brute force,
invariants) and ``tests/test_oracle_mutations.py`` (planted mistakes that the
pins must catch).  The chunked and threaded forms the oracle takes at full
size (``Chunking``) are pinned too, by forcing them on small inputs
(``chunking``).  No function is unpinned.
"""

from .gsa_oracle import (  # noqa: F401
    Chunking,
    Geometry,
    chunking,
    geometry_of,
    spans,
    f64,
    softmax,
    pool,
    compressed_logits,
    compressed_attention,
    guide_scores,
    top_k_blocks,
    top_k_gap,
    selected_keys,
    selected_attention,
    gate,
    combine,
    gsa_layer,
    dense_attention,
    frame_attention,
    sga_sampled,
    sga_key_tokens,
    sga_attention,
    selection_is_valid_top_k,
)
