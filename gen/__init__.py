"""Seeded synthetic inputs for the GenRank hot path.

This package draws data only: sequence structure, ids, timestamps, labels,
embedding tables and projection weights.  It holds none of the method's
arithmetic (no metadata construction, no embedding sums, no attention), so
both the float64 oracle and the CUDA library can take their inputs from it
without sharing any computation.
"""

from .synth import (  # noqa: F401
    CONFIGS,
    Batch,
    Config,
    Model,
    bf16_round,
    config_by_name,
    dense_bias_torch,
    interleave_batch,
    item_rows,
    item_table_torch,
    make_batch,
    make_model,
    make_qkv,
)
