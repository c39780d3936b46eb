"""Pins of the oracle's random streams: published SplitMix64 outputs and the
laws the Rademacher signs and the Gaussian projection must follow."""
import numpy as np
import pytest
from scipy import stats

import oracle


def _golden_ints(path):
    return [int(l) for l in open(path) if l.strip() and not l.startswith("#")]


def test_splitmix64_reference_outputs(golden_dir):
    want = _golden_ints(f"{golden_dir}/splitmix64_seed1234567.txt")
    got = [oracle.splitmix64(1234567, i) for i in range(len(want))]
    assert got == want


def test_rademacher_signs_are_balanced_and_seeded():
    s = oracle.rademacher_signs(1 << 16, 7)
    assert set(np.unique(s)) == {-1, 1}
    # binomial: |#plus - n/2| < 5 sigma
    assert abs((s == 1).sum() - (1 << 15)) < 5 * np.sqrt((1 << 16) / 4)
    assert not np.array_equal(oracle.rademacher_signs(128, 7), oracle.rademacher_signs(128, 8))
    # sign j is a pure function of (seed, j): a prefix of a longer draw
    assert np.array_equal(oracle.rademacher_signs(64, 7), s[:64])


def test_gaussian_draws_are_standard_normal():
    _, g = oracle.gaussian_fp16(512, 512, 3)
    g = g.ravel()
    assert abs(g.mean()) < 5 / np.sqrt(g.size)
    assert abs(g.var() - 1) < 5 * np.sqrt(2 / g.size)
    assert stats.kstest(g, "norm").pvalue > 1e-4
    # third and fourth moments of N(0,1): 0 and 3
    assert abs(stats.skew(g)) < 0.02
    assert abs(stats.kurtosis(g, fisher=False) - 3) < 0.04


def test_gaussian_is_rounded_to_fp16():
    bits, g = oracle.gaussian_fp16(64, 64, 5)
    np.testing.assert_array_equal(bits, g.astype(np.float16).view(np.uint16))


def test_signs_and_projection_use_separate_streams():
    k = oracle.make_constants(128, 2, 1)
    bits, _ = oracle.gaussian_fp16(128, 128, 2)
    np.testing.assert_array_equal(k.S_half, bits)
    np.testing.assert_array_equal(k.delta, oracle.rademacher_signs(128, 1))
