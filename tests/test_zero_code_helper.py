"""The zero-code weight builder used by the outlier parity tests, checked
against the oracle's dequantize: the chosen columns decode to exactly 0 in
every row, every other value is untouched."""
import numpy as np
import pytest

import oracle
import synth
from tests._util import zero_weights_at


@pytest.mark.parametrize("qtype,k", [(oracle.Q8_0, 256), (oracle.Q4_0, 256), (oracle.Q6_K, 512)])
def test_zero_weights_at(qtype, k):
    w = synth.weights(qtype, 9, k, seed=3)
    cols = [0, 1, 15, 16, 17, 31, 33, 100, 127, 128, 150, 200, 255] + ([256, 300, 400, 511] if k > 256 else [])
    z = zero_weights_at(qtype, w, cols)
    a, b = oracle.dequantize(qtype, w, k), oracle.dequantize(qtype, z, k)
    assert np.all(b[:, cols] == 0.0)
    rest = np.setdiff1d(np.arange(k), cols)
    assert np.array_equal(a[:, rest].view(np.uint32), b[:, rest].view(np.uint32))
    # the random weights did not already hold the zero code everywhere
    assert np.count_nonzero(a[:, cols]) > len(cols)
