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


def test_block32_hand_worked_and_round_trip():
    # vector i of a block is bit i of every word: 3 vectors, code of coordinate j of vector v = (v + j) % 4
    codes = (np.arange(3)[:, None] + np.arange(64)[None, :]) % 4
    w = oracle.pack_codes_block32(codes, 2)
    assert w.shape == (1, 2, 64)
    # coordinate 0: codes of vectors 0,1,2 = 0,1,2 -> plane 0 bits 0,1,0 -> 0b010; plane 1 bits 0,0,1 -> 0b100
    assert w[0, 0, 0] == 0b010 and w[0, 1, 0] == 0b100
    rng = np.random.default_rng(1)
    for n in (1, 31, 32, 33, 100):
        c = rng.integers(0, 8, (n, 128))
        np.testing.assert_array_equal(oracle.unpack_codes_block32(oracle.pack_codes_block32(c, 3), 3, 128, n), c)
        bits = rng.integers(0, 2, (n, 64)).astype(np.uint8)
        np.testing.assert_array_equal(oracle.unpack_bits_block32(oracle.pack_bits_block32(bits), 64, n), bits)
    # token and block layouts carry the same bits
    c = rng.integers(0, 4, (64, 128))
    tok = oracle.unpack_codes(oracle.pack_codes(c, 2), 2, 128)
    blk = oracle.unpack_codes_block32(oracle.pack_codes_block32(c, 2), 2, 128, 64)
    np.testing.assert_array_equal(tok, blk)
