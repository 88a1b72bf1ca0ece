"""Float64 CPU oracle for the GenRank hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this package; only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code with the CUDA library.
"""

from .genrank_oracle import (  # noqa: F401
    alibi_slopes,
    attention_bwd,
    attention_bwd_bucketed,
    attention_fwd,
    attention_fwd_bucketed,
    attention_fwd_cached,
    attention_fwd_dense_bias,
    attention_mask,
    bce_loss,
    block_backward,
    block_forward,
    embed_assemble,
    embed_assemble_bwd,
    interleaved_layout,
    pair_time_bucket,
    time_bucket,
    token_metadata,
)
