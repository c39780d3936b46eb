"""Packed cache layout: hand-worked example and round trips."""
import numpy as np

import oracle


def _golden(path):
    rows = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            f = line.split()
            rows[f[0]] = [int(v, 16) for v in f[1:]]
    return rows


def test_hand_worked_packing(golden_dir):
    g = _golden(f"{golden_dir}/pack_example.txt")
    codes = (np.arange(64) % 4)[None, :]
    np.testing.assert_array_equal(oracle.pack_codes(codes, 2).ravel(), np.array(g["codes_words"], np.uint32))
    bits = np.zeros((1, 64), np.uint8)
    bits[0, :8] = 1
    bits[0, 63] = 1
    np.testing.assert_array_equal(oracle.pack_bits(bits).ravel(), np.array(g["qjl_words"], np.uint32))


def test_round_trips():
    rng = np.random.default_rng(0)
    for b in (1, 2, 3, 4):
        for d in (64, 128, 256):
            codes = rng.integers(0, 1 << b, (17, d))
            np.testing.assert_array_equal(oracle.unpack_codes(oracle.pack_codes(codes, b), b, d), codes)
    bits = rng.integers(0, 2, (9, 128)).astype(np.uint8)
    np.testing.assert_array_equal(oracle.unpack_bits(oracle.pack_bits(bits), 128), bits)
