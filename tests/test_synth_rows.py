"""Host copies of sampled query rows (synth.seq_slice_numpy with rows): the oracle reads them
as it reads the whole sequence, without a whole-sequence float64 q being allocated."""
import math

import numpy as np
import pytest

import oracle
import synth


def test_sampled_rows_read_like_the_whole_sequence():
    inp = synth.prefill_inputs([40, 70], 4, 64, 16, seed=3, device="cpu")
    rows = [0, 5, 63, 69]
    part = synth.seq_slice_numpy(inp, 1, rows=rows)
    whole = synth.seq_slice_numpy(inp, 1)
    assert isinstance(part["q"], synth.SampledRows) and part["q"].shape == whole["q"].shape
    for t in rows:
        assert np.array_equal(part["q"][t], whole["q"][t])
        assert np.array_equal(part["q8"][t], whole["q8"][t]) and np.array_equal(part["w"][t], whole["w"][t])
    with pytest.raises(KeyError):
        part["q"][1]  # not sampled: no silent zeros
    sm = 1.0 / math.sqrt(576)
    a = oracle.dsa_prefill_rows(part, 16, sm, rows)
    b = oracle.dsa_prefill_rows(whole, 16, sm, rows)
    for key in ("scores32", "idx", "out", "lse"):
        assert np.array_equal(a[key], b[key]), key
