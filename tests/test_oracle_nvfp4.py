"""Pins for the oracle's NVFP4 block quantizer."""

import os

import numpy as np
import pytest

from oracle import formats, nvfp4, philox


def _golden_blocks(golden_dir):
    cases = []
    with open(os.path.join(golden_dir, "nvfp4_blocks.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, rounding, g, vals, us, scale, codes = (p.strip() for p in line.split("|"))
            cases.append(dict(
                name=name, rounding=rounding, g=float(g),
                v=np.array([float(x) for x in vals.split()], dtype=np.float32),
                fields=None if us == "-" else np.array([int(x) for x in us.split()]),
                scale=int(scale, 16), codes=[int(c, 16) for c in codes.split()]))
    return cases


def test_hand_worked_blocks(golden_dir):
    cases = _golden_blocks(golden_dir)
    assert len(cases) == 7
    for c in cases:
        fields = None if c["fields"] is None else c["fields"][None, :]
        codes, scales = nvfp4.quantize_blocks(c["v"][None, :], c["g"], c["rounding"], fields)
        assert int(scales[0, 0]) == c["scale"], c["name"]
        assert [int(x) for x in codes[0]] == c["codes"], c["name"]


def test_grid_values_are_lossless():
    rng = np.random.default_rng(0)
    mags = formats.E2M1_MAGNITUDES
    for g in (1.0, 0.5, 2.0 ** -10):
        idx = rng.integers(0, 8, size=(64, 32))
        sign = rng.choice([-1.0, 1.0], size=idx.shape)
        s = 2.0 ** rng.integers(-5, 5, size=(64, 2))
        v = (mags[idx] * sign * np.repeat(s, 16, axis=1) * g).astype(np.float32)
        v[:, 0] = 6.0 * s[:, 0] * g          # pin the block max so the scale is exact
        v[:, 16] = 6.0 * s[:, 1] * g
        codes, scales = nvfp4.quantize_blocks(v, g)
        back = nvfp4.dequantize_blocks(codes, scales, g)
        assert np.array_equal(back, v.astype(np.float64))


def test_rn_error_is_at_most_half_a_grid_step():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal((256, 64)) * np.exp(rng.uniform(-4, 4, size=(256, 1)))).astype(np.float32)
    codes, scales = nvfp4.quantize_blocks(v)
    back = nvfp4.dequantize_blocks(codes, scales)
    d = np.repeat(formats.e4m3_decode(scales), 16, axis=1)
    x = np.abs(v / d)
    # local grid spacing of E2M1 around |x| (0.5 below 2, 1 below 4, 2 above)
    step = np.where(x < 2, 0.5, np.where(x < 4, 1.0, 2.0))
    bound = np.maximum(step / 2 * d, (np.abs(v) - 6 * d)) * (1 + 1e-6)
    assert np.all(np.abs(back - v) <= bound + 1e-30)


def test_zero_block_and_tiny_block():
    v = np.zeros((1, 16), dtype=np.float32)
    codes, scales = nvfp4.quantize_blocks(v)
    assert scales[0, 0] == 0 and not codes.any()
    v[0, 3] = 1e-30
    codes, scales = nvfp4.quantize_blocks(v)
    assert scales[0, 0] == 1                  # clamped to 2^-9


def test_non_finite_is_rejected():
    v = np.zeros((1, 16), dtype=np.float32)
    v[0, 5] = np.nan
    with pytest.raises(nvfp4.NonFiniteInput):
        nvfp4.quantize_blocks(v)


def test_sr_up_count_over_all_fields():
    # over the 2^16 equally likely fields an element between grid points rounds up
    # exactly floor(p 2^16) times, p its fractional position
    rng = np.random.default_rng(7)
    F = np.arange(65536)
    for x in np.concatenate([rng.uniform(0, 5.99, 12), [0.25, 0.3, 1.75, 3.999, 4.0000005, 5.5]]).astype(np.float32):
        v = np.zeros((65536, 16), dtype=np.float32)
        v[:, 0] = 6.0                           # scale code 0x38: d = 1, x = v
        v[:, 1] = x
        f = np.zeros((65536, 16), dtype=np.int64)
        f[:, 1] = F
        codes, scales = nvfp4.quantize_blocks(v, 1.0, "sr", f)
        assert np.all(scales == 0x38)
        mags = formats.E2M1_MAGNITUDES[codes[:, 1] & 7]
        grid = formats.E2M1_MAGNITUDES
        lo = grid[np.searchsorted(grid, float(x), "right") - 1]
        hi = grid[np.searchsorted(grid, float(x), "right")]
        p = (float(x) - lo) / (hi - lo)
        assert set(np.unique(mags)) <= {lo, hi}
        assert int(np.sum(mags == hi)) == int(np.floor(p * 65536))


def test_sr_is_unbiased():
    rng = np.random.default_rng(2)
    v = rng.uniform(-5.9, 5.9, size=(1, 16)).astype(np.float32)
    v[0, 0] = 6.0
    acc = np.zeros(16)
    n = 4096
    for seed in range(n):
        codes, scales = nvfp4.quantize_oriented(v, "row", rounding="sr", seed=seed, operand_id=0)
        acc += nvfp4.dequantize_blocks(codes, scales)[0]
    mean = acc / n
    # each element is a two-point variable with spread <= 2 (grid step), sd <= 1
    assert np.all(np.abs(mean - v[0]) <= 4.0 / np.sqrt(n) + 1e-6)


def test_sr_rounds_to_a_neighbour():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((32, 64)).astype(np.float32) * 3
    c_rn, s_rn = nvfp4.quantize_blocks(v)
    c_sr, s_sr = nvfp4.quantize_oriented(v, "row", rounding="sr", seed=5)
    assert np.array_equal(s_rn, s_sr)
    d = np.repeat(formats.e4m3_decode(s_rn), 16, axis=1)
    x = v / d
    mag_sr = formats.E2M1_MAGNITUDES[c_sr & 7]
    lo = formats.E2M1_MAGNITUDES[np.clip(np.searchsorted(formats.E2M1_MAGNITUDES, np.abs(x), "right") - 1, 0, 7)]
    hi = formats.E2M1_MAGNITUDES[np.clip(np.searchsorted(formats.E2M1_MAGNITUDES, np.abs(x), "right"), 0, 7)]
    assert np.all((mag_sr == lo) | (mag_sr == hi))


def test_orientation_and_packing():
    rng = np.random.default_rng(4)
    M = rng.standard_normal((48, 32)).astype(np.float32)
    c_col, s_col = nvfp4.quantize_oriented(M, "col")
    c_rowT, s_rowT = nvfp4.quantize_blocks(np.ascontiguousarray(M.T))
    assert np.array_equal(c_col, c_rowT) and np.array_equal(s_col, s_rowT)
    packed = nvfp4.pack_codes(c_col)
    assert packed.shape == (32, 24)
    assert np.array_equal(packed[:, 0] & 0xF, c_col[:, 0])
    assert np.array_equal(packed[:, 0] >> 4, c_col[:, 1])
    assert np.array_equal(nvfp4.unpack_codes(packed), c_col)


def test_sr_uses_the_orientation_stream():
    rng = np.random.default_rng(6)
    M = rng.standard_normal((16, 16)).astype(np.float32)
    f = philox.sr_fields(9, 2, philox.SR_SUB_COLWISE, 4, 256).reshape(16, 16)
    want, _ = nvfp4.quantize_blocks(np.ascontiguousarray(M.T), 1.0, "sr", f)
    got, _ = nvfp4.quantize_oriented(M, "col", rounding="sr", seed=9, operand_id=2, step=4)
    assert np.array_equal(want, got)


def test_auto_tensor_scale_closed_forms():
    # 6 * 448 = 2688: the bound 2 * amax <= 2688 * g is met with equality at amax = 1344 g
    assert nvfp4.auto_tensor_scale(np.array([[1344.0]])) == 1.0
    assert nvfp4.auto_tensor_scale(np.array([[1344.5]])) == 2.0
    assert nvfp4.auto_tensor_scale(np.array([[-2688.0, 3.0]])) == 2.0
    assert nvfp4.auto_tensor_scale(np.array([[672.0]])) == 0.5
    assert nvfp4.auto_tensor_scale(np.array([[672.5]])) == 1.0
    assert nvfp4.auto_tensor_scale(np.zeros((4, 4))) == 1.0
    assert nvfp4.auto_tensor_scale(np.array([[np.nan, np.inf, 0.0]])) == 1.0
    # 1e-3: bound 7.44e-7 lies between 2^-21 and 2^-20
    assert nvfp4.auto_tensor_scale(np.array([[1e-3]])) == 2.0 ** -20
    # exponent kept in the normal range
    assert nvfp4.auto_tensor_scale(np.array([[1e-41]])) == 2.0 ** -126


def test_auto_tensor_scale_is_the_smallest_admissible_power():
    rng = np.random.default_rng(5)
    for amax in np.exp(rng.uniform(-60, 20, 500)):
        g = nvfp4.auto_tensor_scale(np.array([[amax, -amax / 3]]))
        assert np.log2(g) == np.round(np.log2(g))            # a power of two
        assert 2 * amax <= 2688.0 * g                          # admissible
        assert not 2 * amax <= 2688.0 * g / 2                  # and no smaller one is


def test_auto_tensor_scale_keeps_small_gradients():
    """Gradient-sized data (1e-7) underflows every E4M3 block scale at g = 1; with the
    chosen g the quantization error is the usual NVFP4 level."""
    rng = np.random.default_rng(6)
    M = (rng.standard_normal((32, 64)) * 1e-7).astype(np.float32)
    c1, s1 = nvfp4.quantize_blocks(M, 1.0)
    assert np.all(nvfp4.dequantize_blocks(c1, s1, 1.0) == 0.0) or \
        np.linalg.norm(nvfp4.dequantize_blocks(c1, s1, 1.0) - M) > 0.5 * np.linalg.norm(M)
    g = nvfp4.auto_tensor_scale(M)
    c, s = nvfp4.quantize_blocks(M, g)
    assert np.linalg.norm(nvfp4.dequantize_blocks(c, s, g) - M) < 0.15 * np.linalg.norm(M)


def _pair_decisions(p0, p1, pos0, pos1):
    """Up-rounding decisions of two elements of one 4-group over every value of the
    16 random bits they share: the word's bytes b2:b0 (positions 0, 1) or b3:b1
    (positions 2, 3); the other two bytes are held at zero, which neither decision
    reads.  Returns (up0, up1) boolean arrays over the 2^16 values."""
    v = np.arange(1 << 16, dtype=np.uint64)
    lo, hi = v & np.uint64(0xFF), v >> np.uint64(8)
    shift = 0 if pos0 < 2 else 8
    words = (lo << np.uint64(shift)) | (hi << np.uint64(16 + shift))
    grid = formats.E2M1_MAGNITUDES
    ups = []
    for p, pos in ((p0, pos0), (p1, pos1)):
        a = np.full(v.shape, 1.0 + 0.5 * p)       # between grid points 1 and 1.5
        f = philox.fields_from_words(words, pos)
        ups.append(nvfp4._sr_magnitude(a, f) == 3)
        assert grid[2] == 1.0 and grid[3] == 1.5
    return ups


def test_paired_sr_decisions_are_nearly_independent():
    """Reading R4's field layout gives positions 0 and 1 (and 2 and 3) of a group the
    same 16 bits, one of them bit-reversed.  Each decision is unbiased on its own
    (test_sr_up_count_over_all_fields); this bounds their dependence.  Over all 2^16
    shared bit patterns, at probabilities with at most 8 significant bits the two
    decisions read disjoint bits and are exactly independent; at any probabilities
    the covariance of the two up-roundings stays below 1e-4 (the largest found by a
    search over ~16 million probability pairs is 8.0e-5 at p = 0.646, 0.677, i.e. a
    correlation coefficient of 3.5e-4)."""
    exact = [0.5, 0.25, 0.75, 0.375, 0.9921875, 3 / 256]
    for pos0, pos1 in ((0, 1), (2, 3)):
        for p0 in exact:
            for p1 in exact:
                up0, up1 = _pair_decisions(p0, p1, pos0, pos1)
                t0, t1 = np.floor(p0 * 65536) / 65536, np.floor(p1 * 65536) / 65536
                assert up0.mean() == t0 and up1.mean() == t1
                assert (up0 & up1).mean() == t0 * t1
        worst = [(0.6461639404296875, 0.6769256591796875), (0.3, 0.7), (0.1234, 0.5678), (0.999, 0.001),
                 (1 / 3, 1 / 3), (0.6471895, 0.3565648)]
        for p0, p1 in worst:
            up0, up1 = _pair_decisions(p0, p1, pos0, pos1)
            cov = (up0 & up1).mean() - up0.mean() * up1.mean()
            assert abs(cov) < 1e-4, (p0, p1, cov)


def test_sr_positions_of_different_byte_pairs_read_disjoint_bits():
    """Positions 0/1 read only bytes 0 and 2 of the word, positions 2/3 only bytes 1
    and 3, so decisions across the two pairs are independent for a uniform word."""
    rng = np.random.default_rng(4)
    w = rng.integers(0, 1 << 32, size=4096, dtype=np.uint64)
    m02, m13 = np.uint64(0x00FF00FF), np.uint64(0xFF00FF00)
    w2 = (w & m02) | (rng.integers(0, 1 << 32, size=4096, dtype=np.uint64) & m13)
    w3 = (w & m13) | (rng.integers(0, 1 << 32, size=4096, dtype=np.uint64) & m02)
    for p in (0, 1):
        assert np.array_equal(philox.fields_from_words(w, p), philox.fields_from_words(w2, p))
    for p in (2, 3):
        assert np.array_equal(philox.fields_from_words(w, p), philox.fields_from_words(w3, p))
