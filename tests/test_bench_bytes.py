"""bench.py's algorithmic-byte model of one decode step against the figures
worked out for the two decode layers from the cache layout: 160 B per packed
position outside the vertical-line set, 512 B per FP16 row (vertical lines,
ring, new token), plus the query and output rows; a vertical line's K4V4
record is not algorithmic traffic."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_decode_bytes_1k_layer():
    # L = 1024, W = 128: n = 896 packed, k = 45 lines, T = 1024 before the step
    got = bench.decode_bytes(896, 45, 1024)
    want = 8 * ((896 - 45) * 160 + (45 + 1024 + 1 - 896) * 512) + 2 * 32 * 128 * 2
    assert got == want and abs(got / 1e6 - 1.82) < 0.01


def test_decode_bytes_32k_layer():
    got = bench.decode_bytes(32640, 1632, 32768)
    assert abs(got / 1e6 - 46.92) < 0.01
    # the lines' records would add 1632 x 160 B per kv head
    assert abs((got + 8 * 1632 * 160) / 1e6 - 49.01) < 0.01


def test_k_of_is_the_rational_ceiling():
    assert bench.k_of(32640, 500) == 1632 and bench.k_of(896, 500) == 45 and bench.k_of(0, 500) == 0
