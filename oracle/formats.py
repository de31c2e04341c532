"""Number formats of the hybrid cache and of the prefill's low-precision tiles.

TEST INFRASTRUCTURE ONLY (see the package docstring).

K4V4 (4-bit keys and values).  The pages name the format — "K4V4" for the
non-critical keys and values (HyQuant repository README, Overview item 3 and
the "Mode reference" table; abstract/author comment on the prismix mirror) —
but print no layout.  This library fixes it as follows, and this module is the
definition written out:

* per token row and per head, the D = 128 values are split into 4 groups of
  32 consecutive values;
* for each group: ``mn = min``, ``mx = max`` (exact fp16 values),
  ``scale = fp16_RN( fp32( fp32(mx) - fp32(mn) ) / 15 )`` (two float32 RN
  operations, then RN to fp16), ``zero = mn``;
* each value gets ``q = clamp(rint_even( (fp32(x) - fp32(zero)) / fp32(scale) ), 0, 15)``
  with a float32 RN subtract and a float32 RN divide; when ``scale == 0``
  (constant group, or a range that underflows fp16) every ``q`` is 0;
* two nibbles per byte, low nibble first: byte ``b`` of a row holds
  ``q[2b] | q[2b+1] << 4``.
* the dequantised value is ``zero + q * scale``.

FP8 e4m3 (prefill's quantised tiles; HyQuant README, Overview item 2: most of
prefill's attention matrix products use a low-precision format such as INT8
or FP8).  INT8 (the README's INT8-QK kernels): symmetric per block of 128
positions, ``scale = fp32(amax) / 127`` (1 when amax is 0), a value stored as
``clamp(rint_even(fp32(x) / scale), -127, 127)`` with a float32 RN divide.  The
rounding below is written from the OCP 8-bit floating point specification
(E4M3: bias 7, 3 mantissa bits, no infinities, largest finite 448, smallest
subnormal 2^-9), round-to-nearest-even with saturation to +-448.  Per-block
scaling: one float32 scale per (batch, head, block of 128 positions),
``scale = fp32(amax) / 448`` (1 when amax is 0); a value is stored as
``e4m3_RN_sat( fp32(x) / scale )`` with a float32 RN divide.
"""
from __future__ import annotations

import numpy as np

GROUP = 32
LEVELS = 15
E4M3_MAX = 448.0
FP8_BLOCK = 128


# --------------------------------------------------------------------------- K4V4 and the other widths

BITS = (2, 4, 8)   # per-position code widths of the decode cache (K2 / K4 / K8 and V2 / V4 / V8)


def pack_bits(x16: np.ndarray, bits: int):
    """Pack float16 rows [..., D] with ``bits``-bit codes (2, 4 or 8; README
    Mode reference: the K8V8, K4V2 and K2V4 modes beside K4V4): the K4V4 rule
    with ``2**bits - 1`` levels, ``8 // bits`` codes per byte, lowest bits first.

    Returns ``codes`` uint8 [..., D * bits // 8], ``scale`` and ``zero`` float16 [..., D // 32].
    """
    assert bits in BITS
    levels = (1 << bits) - 1
    x = np.asarray(x16, dtype=np.float16)
    D = x.shape[-1]
    assert D % GROUP == 0
    g = x.reshape(x.shape[:-1] + (D // GROUP, GROUP))
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    span = mx.astype(np.float32) - mn.astype(np.float32)          # float32 RN
    scale = (span / np.float32(levels)).astype(np.float16)          # float32 RN, then RN to fp16
    zero = mn
    diff = g.astype(np.float32) - zero.astype(np.float32)[..., None]  # float32 RN
    s_b = scale.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = diff / s_b                                          # float32 RN
    q = np.where(s_b == 0, 0.0, np.rint(ratio))                      # ties to even
    q = np.clip(q, 0, levels).astype(np.uint32).reshape(x.shape)
    per = 8 // bits
    q = q.reshape(x.shape[:-1] + (D // per, per))
    codes = np.zeros(q.shape[:-1], dtype=np.uint32)
    for i in range(per):
        codes |= q[..., i] << (bits * i)
    return codes.astype(np.uint8), scale, zero


def unpack_bits(codes: np.ndarray, bits: int) -> np.ndarray:
    """uint8 [..., D * bits // 8] -> integer levels [..., D] (lowest bits first)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.uint32)
    per = 8 // bits
    mask = (1 << bits) - 1
    q = np.stack([(c >> (bits * i)) & mask for i in range(per)], axis=-1)
    return q.reshape(c.shape[:-1] + (c.shape[-1] * per,)).astype(np.uint8)


def dequant_bits(codes, scale, zero, bits: int) -> np.ndarray:
    """Dequantised values ``zero + q * scale`` in float64, shape [..., D]."""
    q = unpack_bits(codes, bits).astype(np.float64)
    D = q.shape[-1]
    qg = q.reshape(q.shape[:-1] + (D // GROUP, GROUP))
    x = np.asarray(zero).astype(np.float64)[..., None] + qg * np.asarray(scale).astype(np.float64)[..., None]
    return x.reshape(q.shape)


def dequant_bits_fp16(codes, scale, zero, bits: int) -> np.ndarray:
    """The dequantised values rounded once (RN-even) to float16."""
    return dequant_bits(codes, scale, zero, bits).astype(np.float16)


def pack_k4v4(x16: np.ndarray):
    """Pack float16 rows [..., D] (D a multiple of 32) to K4V4.

    Returns ``codes`` uint8 [..., D // 2], ``scale`` float16 [..., D // 32] and
    ``zero`` float16 [..., D // 32].
    """
    x = np.asarray(x16, dtype=np.float16)
    D = x.shape[-1]
    assert D % GROUP == 0
    g = x.reshape(x.shape[:-1] + (D // GROUP, GROUP))
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    span = mx.astype(np.float32) - mn.astype(np.float32)          # float32 RN
    s32 = span / np.float32(LEVELS)                                 # float32 RN
    scale = s32.astype(np.float16)                                  # RN to fp16
    zero = mn
    diff = g.astype(np.float32) - zero.astype(np.float32)[..., None]  # float32 RN
    s_b = scale.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = diff / s_b                                          # float32 RN
    q = np.rint(ratio)                                              # ties to even
    q = np.where(s_b == 0, 0.0, q)
    q = np.clip(q, 0, LEVELS).astype(np.uint8).reshape(x.shape)
    codes = (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)
    return codes, scale, zero


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """uint8 [..., D//2] -> integer levels uint8 [..., D] (low nibble first)."""
    c = np.asarray(codes, dtype=np.uint8)
    q = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), dtype=np.uint8)
    q[..., 0::2] = c & 0x0F
    q[..., 1::2] = c >> 4
    return q


def dequant_k4v4(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """Dequantised values ``zero + q * scale`` in float64, shape [..., D]."""
    q = unpack_codes(codes).astype(np.float64)
    D = q.shape[-1]
    qg = q.reshape(q.shape[:-1] + (D // GROUP, GROUP))
    x = zero.astype(np.float64)[..., None] + qg * scale.astype(np.float64)[..., None]
    return x.reshape(q.shape)


def dequant_k4v4_fp16(codes, scale, zero) -> np.ndarray:
    """The dequantised values rounded once (RN-even) to float16."""
    return dequant_k4v4(codes, scale, zero).astype(np.float16)


def scale_zero_pairs(scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """Interleave per-group (scale, zero) as float16 [..., D//32, 2] (scale first)."""
    return np.stack([np.asarray(scale, np.float16), np.asarray(zero, np.float16)], axis=-1)


# --------------------------------------------------------------------------- FP8 e4m3

def e4m3_round(x) -> np.ndarray:
    """Nearest OCP E4M3 value (round half to even, saturating at +-448), float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(a)                       # a = m * 2**ex, m in [0.5, 1)
    e = np.maximum(ex.astype(np.float64) - 1.0, -6.0)   # binade exponent, subnormals share -6
    quantum = np.exp2(e - 3.0)                # 3 mantissa bits
    r = np.round(a / quantum) * quantum       # np.round: half to even; a/quantum is exact
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_values() -> np.ndarray:
    """All finite non-negative E4M3 values, decoded from the bit layout (for checks)."""
    vals = []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue                      # S.1111.111 is NaN
            if e == 0:
                vals.append(m / 8.0 * 2.0 ** -6)
            else:
                vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(sorted(set(vals)))


def fp8_block_scales(x16: np.ndarray, block: int = FP8_BLOCK) -> np.ndarray:
    """Per-block scales for x16 [..., L, D]: float32 [..., ceil(L / block)]."""
    x = np.asarray(x16, dtype=np.float16)
    L = x.shape[-2]
    nb = (L + block - 1) // block
    scales = np.empty(x.shape[:-2] + (nb,), dtype=np.float32)
    for i in range(nb):
        amax = np.abs(x[..., i * block:(i + 1) * block, :]).max(axis=(-1, -2)).astype(np.float32)
        s = amax / np.float32(E4M3_MAX)                      # float32 RN
        scales[..., i] = np.where(amax == 0, np.float32(1.0), s)
    return scales


def fp8_quantize(x16: np.ndarray, scales: np.ndarray, block: int = FP8_BLOCK) -> np.ndarray:
    """E4M3 values (float64) of ``fp32(x) / scale`` for x16 [..., L, D]."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float32)
    L = x.shape[-2]
    s = np.repeat(scales, block, axis=-1)[..., :L].astype(np.float32)
    return e4m3_round((x / s[..., None]).astype(np.float32).astype(np.float64))


def fp8_dequant(x8: np.ndarray, scales: np.ndarray, block: int = FP8_BLOCK) -> np.ndarray:
    """Real values represented by FP8 tiles: ``x8 * scale`` in float64."""
    L = x8.shape[-2]
    s = np.repeat(scales.astype(np.float64), block, axis=-1)[..., :L]
    return x8 * s[..., None]


# --------------------------------------------------------------------------- INT8 (symmetric, per block)

INT8_MAX = 127.0


def int8_block_scales(x16: np.ndarray, block: int = FP8_BLOCK) -> np.ndarray:
    """Per-block scales for x16 [..., L, D]: float32 [..., ceil(L / block)], amax / 127 (1 when amax is 0)."""
    x = np.asarray(x16, dtype=np.float16)
    L = x.shape[-2]
    nb = (L + block - 1) // block
    scales = np.empty(x.shape[:-2] + (nb,), dtype=np.float32)
    for i in range(nb):
        amax = np.abs(x[..., i * block:(i + 1) * block, :]).max(axis=(-1, -2)).astype(np.float32)
        scales[..., i] = np.where(amax == 0, np.float32(1.0), amax / np.float32(INT8_MAX))   # float32 RN
    return scales


def int8_quantize(x16: np.ndarray, scales: np.ndarray, block: int = FP8_BLOCK) -> np.ndarray:
    """INT8 codes (as float64 integers) of ``fp32(x) / scale`` for x16 [..., L, D]."""
    x = np.asarray(x16, dtype=np.float16).astype(np.float32)
    L = x.shape[-2]
    s = np.repeat(scales, block, axis=-1)[..., :L].astype(np.float32)
    r = np.rint((x / s[..., None]).astype(np.float32))                 # float32 RN divide, ties to even
    return np.clip(r, -INT8_MAX, INT8_MAX).astype(np.float64)
