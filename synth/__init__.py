"""Seeded synthetic inputs for DSA: shared by the tests, the bench and the oracle checks.

This package holds input recipes only (shapes, distributions, seeds, FP8 encoding of the
inputs, paged-cache layout).  It contains none of the method's arithmetic: no scores, no
selection, no attention.
"""

from .inputs import (  # noqa: F401
    WORKLOADS,
    quantize_e4m3_per_token,
    prefill_inputs,
    prefill_block_inputs,
    decode_inputs,
    exact_prefill_inputs,
    tie_heavy_scores,
    sample_rows,
    seq_slice_numpy,
    decode_seq_numpy,
    SampledRows,
)
