"""The oracle's own binary16 rounding against numpy's (an independent implementation)."""
import numpy as np

import oracle


def test_double_to_half_matches_numpy():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 6, 4000),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
         2.0 ** -14, 2.0 ** -14 * (1 - 2.0 ** -11), 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, np.inf, -np.inf],
    ])
    want = x.astype(np.float16).view(np.uint16)
    got = oracle.double_to_half_bits(x)
    np.testing.assert_array_equal(got, want)


def test_half_to_double_matches_numpy():
    h = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    h = h[(h & 0x7C00) != 0x7C00]  # finite patterns
    np.testing.assert_array_equal(oracle.half_bits_to_double(h), h.view(np.float16).astype(np.float64))
