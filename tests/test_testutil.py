"""The numpy unpacker used to read the GPU's bytes agrees with the oracle's
own unpacking on random codes of every width and both norm modes."""
import numpy as np
import pytest

import oracle as O
from kvq_testutil import compare_codes, unpack_rows


@pytest.mark.parametrize("d", [4, 8, 16, 64, 128, 256])
@pytest.mark.parametrize("L", [2, 3, 7, 64, 128, 255, 256, 4097, 65536])
def test_unpack_rows_matches_oracle(d, L):
    rng = np.random.default_rng(d * L)
    x = (rng.standard_normal((20, d)) * 3).astype(np.float16)
    s = np.where(rng.integers(0, 2, d) == 0, 1, -1).astype(np.int8)
    for mode in (O.MODE_LIN8, O.MODE_LOG4):
        c = O.encode(x, s, L, mode)
        a, n, p = unpack_rows(c.angles, c.norms, c.params, d, L, mode)
        oa, on, _ = O.unpack(c)
        assert np.array_equal(a, oa) and np.array_equal(n, on)
        compare_codes((c.angles, c.norms, c.params), c)


def test_compare_codes_rejects_unflagged_mismatch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 32)).astype(np.float16)
    s = np.ones(32, np.int8)
    c = O.encode(x, s, 128, O.MODE_LIN8)
    bad = c.angles.copy()
    bad[2, 0] ^= 1
    with pytest.raises(AssertionError):
        compare_codes((bad, c.norms, c.params), c)
