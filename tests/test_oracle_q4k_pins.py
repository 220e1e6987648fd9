"""Pins for the oracle's Q4_K decoder ("Red Lite dev15d - DeltaNet gated tail + Q4_K output
projection", section "Q4_K implementation"): the f16 block scales against numpy's binary16 on
every bit pattern, a block packed by hand (tests/golden/q4k_block.txt) whose eight sub-block
scales and mins must come back as stated, the closed form d = 1, dmin = 0, all scales 1 (values
equal the quants, which pins the nibble order), and the block order within a row."""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q4k_block.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            key, *rest = line.split()
            vals[key] = rest
    header = bytes(int(x, 16) for x in vals["header"])
    quants = bytes(17 * (i % 16) for g in range(4) for i in range(32))
    block = np.frombuffer(header + quants, dtype=np.uint8)
    return (float(vals["d"][0]), float(vals["dmin"][0]), [int(x) for x in vals["scales"]],
            [int(x) for x in vals["mins"]], block)


def test_f16_decode_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle._load().oracle_f16_decode(int(b)) for b in bits[::7]], dtype=np.float64)
    r = ref[::7]
    np.testing.assert_array_equal(np.isnan(got), np.isnan(r))
    np.testing.assert_array_equal(got[~np.isnan(r)], r[~np.isnan(r)])


def test_hand_packed_block():
    d, dmin, scales, mins, block = _golden()
    assert block.size == 144
    w = oracle.q4k_dequantize(block.reshape(1, 144), 256)[0]
    for j in range(8):
        for i in range(32):
            q = i % 16
            assert w[32 * j + i] == d * scales[j] * q - dmin * mins[j], (j, i)


def test_unit_scales_give_the_quants():
    rng = np.random.default_rng(5)
    head = np.array([0x00, 0x3C, 0x00, 0x00] + [0x01] * 4 + [0x00] * 4 + [0x01] * 4, dtype=np.uint8)
    qs = rng.integers(0, 256, size=128, dtype=np.uint8)
    w = oracle.q4k_dequantize(np.concatenate([head, qs]).reshape(1, 144), 256)[0]
    for g in range(4):
        np.testing.assert_array_equal(w[64 * g:64 * g + 32], qs[32 * g:32 * g + 32] & 15)
        np.testing.assert_array_equal(w[64 * g + 32:64 * g + 64], qs[32 * g:32 * g + 32] >> 4)


def test_block_order_within_a_row():
    _, _, _, _, block = _golden()
    rng = np.random.default_rng(6)
    other = rng.integers(0, 256, size=144, dtype=np.uint8)
    other[0:4] = [0x00, 0x3C, 0x00, 0x3C]   # d = 1, dmin = 1
    row = np.concatenate([block, other]).reshape(1, 288)
    w = oracle.q4k_dequantize(row, 512)[0]
    np.testing.assert_array_equal(w[:256], oracle.q4k_dequantize(block.reshape(1, 144), 256)[0])
    np.testing.assert_array_equal(w[256:], oracle.q4k_dequantize(other.reshape(1, 144), 256)[0])
    both = oracle.q4k_dequantize(np.stack([np.concatenate([other, block]), row[0]]), 512)
    np.testing.assert_array_equal(both[0, :256], w[256:])
    np.testing.assert_array_equal(both[1], w)
