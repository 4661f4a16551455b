"""E2M1 and E4M3 number formats, encoded by exhaustive nearest search.

The Metis notes ("Metis: Training LLMs with FP4 Quantization", 研究背景 /
现有痛点 and 训练策略) fix NVFP4 as 4-bit E2M1 elements in blocks of 16 with
one 8-bit floating-point scale per block; the scale format is E4M3 (the OCP
"fn" variant: no infinities, 0x7F/0xFF are NaN, largest finite 448).

E2M1 (1 sign, 2 exponent, 1 mantissa bit, bias 1) has the magnitudes
{0, 0.5, 1, 1.5, 2, 3, 4, 6} for codes 0..7; bit 3 is the sign.

Readings (the pages are silent on rounding details):
* round to nearest, ties to the even code (the code whose lowest bit is 0);
* saturate: anything beyond the largest finite value encodes as that value;
* the sign bit is kept, so -0 and small negatives that round to zero encode
  as 0x8.

Pins (tests/test_oracle_formats.py): every code decodes to its closed-form
value and re-encodes to itself; every midpoint between neighbours goes to the
even code; the tables match the format definitions bit by bit.
"""

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def e4m3_positive_table():
    """Values of E4M3 codes 0..126 (all non-negative finite codes), ascending."""
    vals = np.zeros(127, dtype=np.float64)
    for code in range(127):
        e = code >> 3
        m = code & 7
        if e == 0:
            vals[code] = m * 2.0 ** -9          # subnormal: m/8 * 2^(1-7)
        else:
            vals[code] = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_TABLE = e4m3_positive_table()


def e2m1_decode(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag)


def _nearest_even(absx, table):
    """Index of the nearest table entry to each |x|; ties go to the even index.

    Exhaustive: distances to every table entry are formed and compared.
    ``absx`` is float64 and every table value is exact in float64, so the
    distances and the tie test are exact for fp32 inputs.
    """
    absx = np.asarray(absx, dtype=np.float64)
    out = np.empty(absx.shape, dtype=np.int64)
    flat = absx.reshape(-1)
    res = out.reshape(-1)
    chunk = max(1, (1 << 22) // len(table))
    idx = np.arange(len(table))
    for s in range(0, flat.size, chunk):
        v = flat[s:s + chunk, None]
        d = np.abs(v - table[None, :])
        dmin = d.min(axis=1, keepdims=True)
        cand = d == dmin
        # among equally near entries prefer the even index
        even_cand = cand & (idx[None, :] % 2 == 0)
        pick = np.where(even_cand.any(axis=1), even_cand.argmax(axis=1), cand.argmax(axis=1))
        res[s:s + chunk] = pick
    return out


def e2m1_encode_rn(x):
    """fp32/fp64 values -> E2M1 codes (uint8), RN-even, saturating, sign kept."""
    x = np.asarray(x, dtype=np.float64)
    absx = np.minimum(np.abs(x), E2M1_MAX)
    code = _nearest_even(absx, E2M1_MAGNITUDES).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 3
    return code | sign


def e4m3_encode_rn(x):
    """Non-negative values -> E4M3 codes (uint8), RN-even, satfinite."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(x < 0) or np.any(np.isnan(x)):
        raise ValueError("E4M3 scale encoder takes non-negative finite values")
    clipped = np.minimum(x, E4M3_MAX)
    return _nearest_even(clipped, E4M3_TABLE).astype(np.uint8)


def e4m3_decode(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    if np.any((codes & 0x7F) == 0x7F):
        raise ValueError("E4M3 NaN code")
    mag = E4M3_TABLE[codes & 0x7F]
    return np.where(codes & 0x80, -mag, mag)
