"""NVFP4 block quantizer Q_b.

Source: "Metis: Training LLMs with FP4 Quantization" (papernotes.org notes),
研究背景 / 现有痛点 (NVFP4: E2M1 values, block size 16, one FP8 scale per block
chosen from the block maximum) and 训练策略 (W4A4G4 in E2M1, stochastic
rounding on by default).

A matrix is quantized in one orientation: it is viewed as ``outer x inner``
and every run of 16 consecutive elements along ``inner`` is one block.  For a
block v with decode tensor scale g (a power of two):

1. amax = max |v|                                   (exact)
2. s    = E4M3_RN( fl32(amax / fl32(6 g)) )         (IEEE fp32 division)
3. if amax > 0 and s == 0:  s = 2^-9                (smallest E4M3 value)
4. if amax == 0: scale code 0 and every element code +0
5. d    = fl32(s * g);  r = fl32(1 / d)             (IEEE fp32 reciprocal)
6. x    = fl32(v * r)
7. code = E2M1_RN(x)  or, with stochastic rounding, the SR rule below
8. decoded value = e2m1(code) * s * g

Stochastic rounding (R4 of the build's readings): with a = |x|, if a >= 6 the
magnitude is 6; otherwise lo <= a < hi are the neighbouring E2M1 magnitudes,
p = (a - lo) / (hi - lo) (exact: a - lo is exact by Sterbenz, hi - lo is a
power of two) and the magnitude rounds up to hi iff

    floor(p * 2^16) + F >= 2^16,

F being the element's 16-bit random field from ``philox.sr_fields`` (so the
chance of rounding up is floor(p * 2^16) / 2^16: unbiased to within 2^-16 of a
grid step).  The sign of x is kept, so a negative value that rounds to zero
gives -0.  Scales are always rounded to nearest.

Readings that go beyond the pages: the per-tensor decode scale g (1.0 for
residuals unless the caller sets one or asks for ``auto_tensor_scale``), the
reciprocal multiply in step 5-6, and the SR random-field layout.

Pins (tests/test_oracle_nvfp4.py): round trips of values already on the
grid, the scale rule against hand-computed blocks, dequantization error
bounded by half a grid step, SR: the exact count of up-roundings over all
2^16 fields, unbiasedness over many seeds, a hand-worked block; the all-zero
block, saturation, and the packed layout.
"""

import numpy as np

from . import formats, philox

BLOCK = 16


class NonFiniteInput(ValueError):
    pass


E2M1_MAX = 6.0
E4M3_MAX = 448.0


def auto_tensor_scale(M):
    """The decode tensor scale g chosen from the data (reading R1b): the smallest
    power of two g with 2 * amax <= 6 * 448 * g, amax = max |M| over the finite
    entries (so the largest block of M, or of a residual of M up to twice its size,
    gets an E4M3 block scale of at most 448); 1.0 when M has no nonzero finite entry;
    the exponent is kept within the normal fp32 range [-126, 127].

    Written as the definition: start from a power of two at or above the bound and
    step down while the next smaller one still satisfies it."""
    A = np.abs(np.asarray(M, dtype=np.float64))
    A = A[np.isfinite(A)]
    amax = float(A.max()) if A.size else 0.0
    if amax == 0.0:
        return 1.0
    bound = 2.0 * amax / (E2M1_MAX * E4M3_MAX)
    e = int(np.ceil(np.log2(bound))) + 1
    while e > -126 and bound <= 2.0 ** (e - 1):
        e -= 1
    while bound > 2.0 ** e:
        e += 1
    return float(2.0 ** min(max(e, -126), 127))


def _scale_codes(amax, g):
    six_g = np.float32(6.0) * np.float32(g)
    target = (amax.astype(np.float32) / six_g).astype(np.float32)
    codes = formats.e4m3_encode_rn(target.astype(np.float64))
    codes = np.where((amax > 0) & (codes == 0), np.uint8(1), codes).astype(np.uint8)
    return codes


def _sr_magnitude(a, fields):
    """Stochastic rounding of magnitudes a in [0, 6) onto the E2M1 grid (index of the result)."""
    grid = formats.E2M1_MAGNITUDES
    lo_idx = np.searchsorted(grid, a, side="right") - 1       # grid[lo_idx] <= a < grid[lo_idx+1]
    lo = grid[lo_idx]
    hi = grid[lo_idx + 1]
    p = (a - lo) / (hi - lo)
    up = np.floor(p * 65536.0) + np.asarray(fields, dtype=np.float64) >= 65536.0
    return np.where(up, lo_idx + 1, lo_idx)


def quantize_blocks(M, g=1.0, rounding="rn", fields=None):
    """Quantize ``M`` (outer x inner, fp32 values) with 16-blocks along inner.

    Returns (codes, scale_codes): codes is uint8 (outer x inner) holding one
    E2M1 code per element (sign in bit 3); scale_codes is uint8
    (outer x inner/16) holding E4M3 codes.
    """
    M = np.asarray(M, dtype=np.float32)
    outer, inner = M.shape
    if inner % BLOCK:
        raise ValueError("inner dimension must be a multiple of 16")
    if not np.all(np.isfinite(M)):
        raise NonFiniteInput("non-finite value in quantizer input")
    g = np.float32(g)
    blocks = M.reshape(outer, inner // BLOCK, BLOCK)
    amax = np.abs(blocks).max(axis=2)
    s_codes = _scale_codes(amax, g)
    s_val = formats.e4m3_decode(s_codes).astype(np.float32)
    d = (s_val * g).astype(np.float32)
    zero_block = s_codes == 0
    d_safe = np.where(zero_block, np.float32(1.0), d)
    r = (np.float32(1.0) / d_safe).astype(np.float32)
    x = (blocks * r[:, :, None]).astype(np.float32)
    if rounding == "rn":
        codes = formats.e2m1_encode_rn(x.astype(np.float64))
    elif rounding == "sr":
        if fields is None:
            raise ValueError("stochastic rounding needs random fields")
        fields = np.asarray(fields, dtype=np.int64).reshape(outer, inner // BLOCK, BLOCK)
        a = np.abs(x.astype(np.float64))
        saturated = a >= 6.0
        mag_idx = np.where(saturated, 7, _sr_magnitude(np.where(saturated, 0.0, a), fields))
        codes = (mag_idx.astype(np.uint8) | (np.signbit(x).astype(np.uint8) << 3))
    else:
        raise ValueError(rounding)
    codes = np.where(zero_block[:, :, None], np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(outer, inner), s_codes


def dequantize_blocks(codes, scale_codes, g=1.0):
    codes = np.asarray(codes, dtype=np.uint8)
    outer, inner = codes.shape
    vals = formats.e2m1_decode(codes).reshape(outer, inner // BLOCK, BLOCK)
    s = formats.e4m3_decode(scale_codes)
    return (vals * s[:, :, None] * float(g)).reshape(outer, inner)


def pack_codes(codes):
    """(outer x inner) codes -> (outer x inner/2) bytes, even element in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed):
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def quantize_oriented(M, orientation, g=1.0, rounding="rn", seed=0, operand_id=0,
                      step=0, sr_sub=None):
    """Quantize an r x c matrix row-wise (blocks along c) or column-wise.

    Column-wise quantization is row-wise quantization of M^T, so both return
    ``outer x inner`` codes with inner the blocked (contraction) dimension.
    SR fields follow the blocked-contiguous element order e = i*inner + j
    of the oriented view, from sub-stream ``sr_sub`` (default: 0 for
    row-wise, 1 for column-wise).
    """
    M = np.asarray(M, dtype=np.float32)
    view = M if orientation == "row" else M.T
    view = np.ascontiguousarray(view)
    fields = None
    if rounding == "sr":
        if sr_sub is None:
            sr_sub = philox.SR_SUB_ROWWISE if orientation == "row" else philox.SR_SUB_COLWISE
        fields = philox.sr_fields(seed, operand_id, sr_sub, step, view.size).reshape(view.shape)
    return quantize_blocks(view, g, rounding, fields)
