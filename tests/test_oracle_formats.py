"""Pins for the E2M1 / E4M3 tables and encoders of the oracle."""

import numpy as np
import pytest
import torch

from oracle import formats


def test_e2m1_table_from_bit_fields():
    # E2M1: 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is subnormal.
    for code in range(8):
        e, m = (code >> 1) & 3, code & 1
        val = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
        assert formats.E2M1_MAGNITUDES[code] == val
    assert list(formats.E2M1_MAGNITUDES) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e2m1_round_trip_every_code():
    codes = np.arange(16, dtype=np.uint8)
    vals = formats.e2m1_decode(codes)
    # -0 (code 8) decodes to -0.0 and must re-encode to 8
    vals = np.where(codes == 8, -0.0, vals)
    assert list(formats.e2m1_encode_rn(vals)) == list(codes)


def test_e2m1_midpoints_go_to_even_code():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0, 2, 2, 4, 4, 6, 6]
    assert list(formats.e2m1_encode_rn(mids)) == want
    assert list(formats.e2m1_encode_rn([-m for m in mids])) == [8 | w for w in want]


def test_e2m1_nearest_off_midpoint_and_saturation():
    eps = 1e-6
    assert list(formats.e2m1_encode_rn([0.25 + eps, 0.75 - eps, 5 + eps])) == [1, 1, 7]
    assert list(formats.e2m1_encode_rn([6.0, 7.0, 1e9, -1e9])) == [7, 7, 7, 15]


def test_e4m3_table_anchors():
    t = formats.E4M3_TABLE
    assert t[0] == 0 and t[1] == 2.0 ** -9 and t[7] == 7 * 2.0 ** -9
    assert t[8] == 2.0 ** -6              # smallest normal
    assert t[0x38] == 1.0 and t[0x3F] == 1.875 and t[0x40] == 2.0
    assert t[0x7E] == 448.0               # largest finite
    assert np.all(np.diff(t) > 0)


def test_e4m3_matches_torch_float8_e4m3fn_on_a_dense_sweep():
    # torch.float8_e4m3fn rounds to nearest even; compare within its finite range
    x = np.concatenate([np.linspace(0, 460, 200001), np.geomspace(1e-6, 460, 200001)])
    x32 = x.astype(np.float32)
    ours = formats.e4m3_encode_rn(x32.astype(np.float64))
    ref = torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(formats.e4m3_decode(codes), ref)


def test_e4m3_saturates_and_rejects_bad_input():
    assert list(formats.e4m3_encode_rn([448.0, 464.0, 1e6])) == [0x7E] * 3
    with pytest.raises(ValueError):
        formats.e4m3_encode_rn([-1.0])
    with pytest.raises(ValueError):
        formats.e4m3_decode([0x7F])
