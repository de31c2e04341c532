"""Pins for the oracle's number formats (K4V4 pack/dequant, FP8 e4m3), CPU only.

Each check comes from outside the oracle's own code: hand-worked groups,
brute-force searches over the levels, the OCP E4M3 bit layout, and the
correctly rounded float16 conversion of Python's ``struct`` module.
"""
import os
import struct
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats

GOLD = os.path.join(os.path.dirname(__file__), "golden", "k4v4_groups.txt")


def _load_groups():
    rows = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, vals, sc, ze, codes = [t.strip() for t in line.split("|")]
        x = np.array([float(t) for t in vals.split()], dtype=np.float64)
        assert len(x) == 32 and np.all(x.astype(np.float16).astype(np.float64) == x), name
        rows.append((name, x.astype(np.float16), int(sc, 16), int(ze, 16), bytes.fromhex(codes.replace(" ", ""))))
    return rows


@pytest.mark.parametrize("name,x,scale_bits,zero_bits,codes", _load_groups())
def test_k4v4_hand_groups(name, x, scale_bits, zero_bits, codes):
    c, s, z = formats.pack_k4v4(x)
    assert c.tobytes() == codes, name
    assert int(s.view(np.uint16)[0]) == scale_bits, name
    assert int(z.view(np.uint16)[0]) == zero_bits, name


def test_k4v4_group_boundaries_and_nibble_order():
    # four groups with different ranges: each group gets its own scale/zero
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(lo, hi, 32) for lo, hi in ((0, 1), (-8, -4), (100, 101), (-1, 1))]).astype(np.float16)
    c, s, z = formats.pack_k4v4(x)
    for g in range(4):
        xg = x[32 * g:32 * g + 32]
        assert z[g] == xg.min()
        c1, s1, z1 = formats.pack_k4v4(xg)
        assert c1.tobytes() == c[16 * g:16 * g + 16].tobytes() and s1[0] == s[g]
    q = formats.unpack_codes(c)
    assert np.all(q[0::2] == (c & 15)) and np.all(q[1::2] == (c >> 4))


def test_k4v4_levels_are_nearest():
    """Brute force: every code is a nearest of the 16 levels (up to fp32 rounding of the ratio)."""
    rng = np.random.default_rng(1)
    for trial in range(300):
        lo = rng.normal() * 4
        span = abs(rng.normal()) * 3 + 1e-3
        x = (lo + span * rng.random(32)).astype(np.float16)
        c, s, z = formats.pack_k4v4(x)
        q = formats.unpack_codes(c).astype(np.int64)
        sc = float(s[0]); ze = float(z[0])
        levels = ze + np.arange(16) * sc
        err = np.abs(x.astype(np.float64)[:, None] - levels[None, :])
        best = err.min(axis=1)
        chosen = err[np.arange(32), q]
        # the divide is one float32 rounding: allow a relative 2^-22 of the level spacing
        assert np.all(chosen <= best + sc * 2.0 ** -20), trial
        assert q.min() == 0


def test_k4v4_roundtrip_bound():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128)).astype(np.float16)
    c, s, z = formats.pack_k4v4(x)
    xh = formats.dequant_k4v4(c, s, z)
    bound = np.repeat(s.astype(np.float64), 32, axis=-1) * 0.5 * (1 + 2.0 ** -9)
    assert np.all(np.abs(xh - x.astype(np.float64)) <= bound + 1e-12)
    # the top level never overshoots the group's span by more than the fp16 rounding of scale
    top = z.astype(np.float64) + 15 * s.astype(np.float64)
    mx = x.reshape(64, 4, 32).max(axis=-1).astype(np.float64)
    assert np.all(np.abs(top - mx) <= 15 * s.astype(np.float64) * 2.0 ** -11 + 1e-12)


def test_k4v4_scale_is_fp32_then_fp16():
    # independent recomputation of the scale with exact rationals and struct's
    # correctly rounded fp32/fp16 conversions
    rng = np.random.default_rng(3)
    for _ in range(200):
        a, b = np.sort(rng.standard_normal(2) * rng.choice([1e-3, 1, 30])).astype(np.float16)
        x = np.full(32, a, np.float16)
        x[7] = b
        _, s, _ = formats.pack_k4v4(x)
        span32 = struct.unpack("<f", struct.pack("<f", float(Fraction(float(b)) - Fraction(float(a)))))[0]
        q32 = struct.unpack("<f", struct.pack("<f", float(Fraction(span32) / 15)))[0]
        want = struct.unpack("<e", struct.pack("<e", q32))[0]
        assert float(s[0]) == want


def test_dequant_fp16_is_single_rounding():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((32, 128)) * 7).astype(np.float16)
    c, s, z = formats.pack_k4v4(x)
    got = formats.dequant_k4v4_fp16(c, s, z)
    q = formats.unpack_codes(c).reshape(32, 4, 32)
    for r in range(32):
        for g in range(4):
            for i in range(32):
                exact = Fraction(float(z[r, g])) + int(q[r, g, i]) * Fraction(float(s[r, g]))
                assert float(got[r, g * 32 + i]) == struct.unpack("<e", struct.pack("<e", float(exact)))[0]


# ------------------------------------------------------------------ E4M3

def test_e4m3_table_from_bit_layout():
    v = formats.e4m3_values()
    assert len(v) == 127                      # 128 codes minus the NaN pattern
    assert v[0] == 0 and v[1] == 2.0 ** -9 and v[-1] == 448.0
    assert 2.0 ** -6 in v and 1.75 * 2 ** 8 == 448.0
    assert np.all(formats.e4m3_round(v) == v)
    assert np.all(formats.e4m3_round(-v) == -v)


def _nearest_even_by_table(x):
    v = formats.e4m3_values()
    a = abs(x)
    if a >= 448:
        return np.copysign(448.0, x)
    i = np.searchsorted(v, a)
    lo, hi = v[i - 1] if i > 0 else v[0], v[min(i, len(v) - 1)]
    if a - lo < hi - a:
        r = lo
    elif hi - a < a - lo:
        r = hi
    else:   # tie: the code with an even mantissa (even index in the sorted table)
        r = lo if (i - 1) % 2 == 0 else hi
    return np.copysign(r, x)


def test_e4m3_round_matches_table_search():
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-3, 2.7, 3000)])
    v = formats.e4m3_values()
    mids = (v[1:] + v[:-1]) / 2
    xs = np.concatenate([xs, mids, -mids, [460.0, 464.0, 470.0, 1e6, 2.0 ** -10, 3 * 2.0 ** -11]])
    got = formats.e4m3_round(xs)
    want = np.array([_nearest_even_by_table(x) for x in xs])
    assert np.array_equal(got, want)
    assert formats.e4m3_round(2.0 ** -10) == 0.0 and formats.e4m3_round(3 * 2.0 ** -11) == 2.0 ** -9
    assert formats.e4m3_round(464.0) == 448.0 and formats.e4m3_round(-1e9) == -448.0


def test_fp8_block_scales_and_quantize():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((2, 300, 16)) * 3).astype(np.float16)
    x[1, 128:256] = 0
    s = formats.fp8_block_scales(x)
    assert s.shape == (2, 3)
    for b in range(2):
        for k in range(3):
            blk = x[b, 128 * k:128 * k + 128].astype(np.float32)
            amax = np.abs(blk).max()
            assert s[b, k] == (np.float32(1) if amax == 0 else np.float32(amax) / np.float32(448))
    q = formats.fp8_quantize(x, s)
    assert np.abs(q).max() <= 448 and np.all(formats.e4m3_round(q) == q)
    # the block maximum maps to exactly +-448 (amax/scale rounds back to 448)
    for b in range(2):
        for k in range(3):
            if np.abs(x[b, 128 * k:128 * k + 128]).max() > 0:
                assert np.abs(q[b, 128 * k:128 * k + 128]).max() == 448.0
    back = formats.fp8_dequant(q, s)
    rel = np.abs(back - x.astype(np.float64)) / np.maximum(np.abs(x.astype(np.float64)), 1e-3)
    big = np.abs(x.astype(np.float64)) > np.repeat(s, 128, axis=-1)[..., :300, None] * 2.0 ** -6 * 8
    assert np.all(rel[big] <= 2.0 ** -4 + 1e-6)


# ------------------------------------------------------------------ the 2-bit and 8-bit widths

GOLD_BITS = os.path.join(os.path.dirname(__file__), "golden", "kv_bits_groups.txt")


def _load_bit_groups():
    rows = []
    for line in open(GOLD_BITS):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, bits, vals, sc, ze, codes = [t.strip() for t in line.split("|")]
        x = np.array([float(t) for t in vals.split()], dtype=np.float64)
        assert len(x) == 32 and np.all(x.astype(np.float16).astype(np.float64) == x), name
        rows.append((name, int(bits), x.astype(np.float16), int(sc, 16), int(ze, 16), bytes.fromhex(codes.replace(" ", ""))))
    return rows


@pytest.mark.parametrize("name,bits,x,scale_bits,zero_bits,codes", _load_bit_groups())
def test_bits_hand_groups(name, bits, x, scale_bits, zero_bits, codes):
    c, s, z = formats.pack_bits(x, bits)
    assert c.tobytes() == codes, name
    assert int(s.view(np.uint16)[0]) == scale_bits, name
    assert int(z.view(np.uint16)[0]) == zero_bits, name
    q = formats.unpack_bits(c, bits)
    # unpacking reads the codes back lowest bits first
    per = 8 // bits
    for j in range(32):
        assert q[j] == (codes[j // per] >> (bits * (j % per))) & ((1 << bits) - 1)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_bits_levels_are_nearest(bits):
    """Brute force over the 2^bits levels: every code is a nearest level of its
    value (up to the float32 rounding of the ratio), and dequantisation is
    zero + q * scale exactly."""
    levels = (1 << bits) - 1
    rng = np.random.default_rng(bits)
    for trial in range(200):
        lo = rng.normal() * 4
        span = abs(rng.normal()) * 3 + 1e-3
        x = (lo + span * rng.random(32)).astype(np.float16)
        c, s, z = formats.pack_bits(x, bits)
        q = formats.unpack_bits(c, bits).astype(np.int64)
        sc, ze = float(s[0]), float(z[0])
        assert ze == float(x.min())
        assert sc == float(np.float16(np.float32(np.float32(x.max()) - np.float32(x.min())) / np.float32(levels)))
        for j in range(32):
            cand = [abs(float(x[j]) - (ze + L * sc)) for L in range(levels + 1)]
            best = min(cand)
            assert cand[q[j]] <= best + sc * 1e-6 + 1e-12, (bits, trial, j)
        deq = formats.dequant_bits(c, s, z, bits)
        assert np.array_equal(deq, ze + q * sc)


def test_bits_four_is_k4v4_and_sizes():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 128)).astype(np.float16)
    a, b = formats.pack_k4v4(x), formats.pack_bits(x, 4)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))
    for bits in (2, 4, 8):
        c, s, z = formats.pack_bits(x, bits)
        assert c.shape == (3, 128 * bits // 8) and s.shape == z.shape == (3, 4)


# ------------------------------------------------------------------ INT8 (prefill's INT8-QK format)

def test_int8_block_hand_examples():
    """Worked by hand: a block whose amax is 127 has scale exactly 1, so codes
    are the values rounded half to even; a block with amax 254 has scale 2."""
    x = np.zeros((128, 128), np.float16)
    x[0, :8] = [0.5, 1.5, 2.5, -0.5, -1.5, 127, -127, 3.25]
    s = formats.int8_block_scales(x)
    assert s.tolist() == [1.0]
    q = formats.int8_quantize(x, s)
    assert q[0, :8].tolist() == [0, 2, 2, 0, -2, 127, -127, 3]
    y = np.zeros((200, 128), np.float16)
    y[5, 3] = 254
    y[6, 0:4] = [3, 5, -7, 1]
    y[150, 0] = -2.0                        # second block: amax 2, scale 2/127
    s = formats.int8_block_scales(y)
    assert s[0] == 2.0 and s[1] == np.float32(2.0) / np.float32(127.0)
    q = formats.int8_quantize(y, s)
    assert q[6, 0:4].tolist() == [2, 2, -4, 0] and q[5, 3] == 127 and q[150, 0] == -127
    assert formats.int8_block_scales(np.zeros((10, 128), np.float16)).tolist() == [1.0]


def test_int8_codes_are_nearest_and_bounded():
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((300, 128)) * rng.uniform(0.1, 50, (300, 1))).astype(np.float16)
    s = formats.int8_block_scales(x)
    q = formats.int8_quantize(x, s)
    assert np.all(np.abs(q) <= 127) and np.all(q == np.round(q))
    for blk in range(len(s)):
        rows = slice(128 * blk, 128 * (blk + 1))
        r = x[rows].astype(np.float64) / float(s[blk])
        assert np.all(np.abs(q[rows] - r) <= 0.5 + 1e-5)
        amax = np.abs(x[rows]).max()
        assert np.abs(q[rows]).max() == 127 or amax == 0
