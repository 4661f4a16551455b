"""Pins for the oracle's Philox4x32-10 and its derived streams."""

import os

import numpy as np
import pytest

from oracle import philox


def _kat_rows(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            ctr, key, out = (part.split() for part in line.split("|"))
            rows.append(([int(x, 16) for x in ctr], [int(x, 16) for x in key],
                         [int(x, 16) for x in out]))
    return rows


def test_known_answer_vectors(golden_dir):
    rows = _kat_rows(golden_dir)
    assert len(rows) == 3
    for ctr, key, out in rows:
        got = philox.philox4x32_10(*ctr, *key)
        assert [int(w) for w in got] == out


def test_vectorised_matches_scalar():
    q = np.array([0, 1, 2, 12345, 2**32 + 7], dtype=np.uint64)
    words = philox.stream_words(0x1234_5678_9ABC_DEF0, 0x0213, 5, q)
    for i, qi in enumerate(q):
        single = philox.philox4x32_10(int(qi) & 0xFFFFFFFF, int(qi) >> 32, 0x0213, 5,
                                      0x9ABCDEF0, 0x12345678)
        assert [int(w) for w in single] == [int(w) for w in words[i]]


def test_element_words_layout():
    w = philox.element_words(7, 0x31, 2, 10)
    calls = philox.stream_words(7, 0x31, 2, np.arange(3, dtype=np.uint64))
    for e in range(10):
        assert int(w[e]) == int(calls[e >> 2][e & 3])


def test_sr_field_layout():
    # element e: counter e >> 4, word (e >> 2) & 3, position e & 3 of the word's group
    n = 40
    f = philox.sr_fields(3, 1, philox.SR_SUB_COLWISE, 9, n)
    calls = philox.stream_words(3, philox.tag(1, philox.PURPOSE_SR, philox.SR_SUB_COLWISE), 9,
                                np.arange(3, dtype=np.uint64))
    for e in range(n):
        word = int(calls[e >> 4][(e >> 2) & 3])
        assert int(f[e]) == int(philox.fields_from_words(np.uint64(word), e & 3))
    assert np.all((f >= 0) & (f < 65536))
    at = philox.sr_fields_at(3, 1, philox.SR_SUB_COLWISE, 9, np.array([39, 0, 17]))
    assert [int(x) for x in at] == [int(f[39]), int(f[0]), int(f[17])]


def test_sr_fields_of_a_word_by_hand():
    # W = 0x12345678: b0 = 0x78, b1 = 0x56, b2 = 0x34, b3 = 0x12
    # position 0: b2:b0 = 0x3478; 1: 0x3478 bit-reversed = 0x1E2C;
    # position 2: b3:b1 = 0x1256; 3: 0x1256 bit-reversed = 0x6A48
    w = np.uint64(0x12345678)
    got = [int(philox.fields_from_words(w, p)) for p in range(4)]
    assert got == [0x3478, 0x1E2C, 0x1256, 0x6A48]


def test_sr_fields_are_uniform_per_position():
    # 2^14 groups: the high byte of every position's field is uniform (chi-square,
    # 255 dof, mean 255, sd ~22.6)
    f = philox.sr_fields(11, 0, philox.SR_SUB_ROWWISE, 0, 1 << 16).reshape(-1, 4)
    for p in range(4):
        counts = np.bincount((f[:, p] >> 8).astype(np.int64), minlength=256)
        expected = f.shape[0] / 256
        chi2 = float(np.sum((counts - expected) ** 2 / expected))
        assert 150 < chi2 < 380, p


def test_uniformity_chi_square():
    # 2^16 draws of the low byte: chi-square with 255 dof, mean 255, sd ~22.6
    w = philox.element_words(11, philox.tag(0, philox.PURPOSE_SR), 0, 1 << 16)
    counts = np.bincount((w & np.uint64(0xFF)).astype(np.int64), minlength=256)
    expected = (1 << 16) / 256
    chi2 = float(np.sum((counts - expected) ** 2 / expected))
    assert 150 < chi2 < 380


def test_streams_are_distinct():
    a = philox.element_words(1, philox.tag(0, philox.PURPOSE_SAMPLE), 0, 64)
    b = philox.element_words(1, philox.tag(0, philox.PURPOSE_OMEGA), 0, 64)
    c = philox.element_words(1, philox.tag(1, philox.PURPOSE_SAMPLE), 0, 64)
    d = philox.element_words(1, philox.tag(0, philox.PURPOSE_SAMPLE), 1, 64)
    assert len({a.tobytes(), b.tobytes(), c.tobytes(), d.tobytes()}) == 4


def test_tag_fields():
    assert philox.tag(2, philox.PURPOSE_SR, 3) == (2 << 8) | (3 << 4) | 3
    with pytest.raises(TypeError):
        philox.tag()
