"""Philox4x32-10 and the random streams the method draws from.

Generator: Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as
1, 2, 3" (SC'11), the 4x32 variant with 10 rounds.  One call maps a 128-bit
counter (c0..c3) and a 64-bit key (k0, k1) to four 32-bit words.  A round is

    (hi0, lo0) = M0 * c0        (full 64-bit product split in two halves)
    (hi1, lo1) = M1 * c2
    c' = (hi1 ^ c1 ^ k0,  lo1,  hi0 ^ c3 ^ k1,  lo0)

and the key is bumped by the Weyl constants (W0, W1) between rounds.

The Metis notes ("Metis: Training LLMs with FP4 Quantization", 关键设计 2 and
训练策略) draw randomness in three places: the sparse row sample, the Gaussian
test matrix Omega and stochastic rounding.  The pages fix no generator; both
this oracle and the CUDA library implement this one generator from its
published definition, with the stream layout below:

    key     = (seed & 0xffffffff, seed >> 32)
    counter = (q & 0xffffffff, q >> 32, tag, step)
    tag     = operand_id << 8 | purpose << 4 | sub

``purpose`` is SAMPLE, OMEGA or SR; ``sub`` separates streams of one purpose
(for SR: the residual's row-wise and column-wise quantization, and the two
factor matrices).

Stochastic rounding draws 16 random bits per element.  A 32-bit word serves a
group of four consecutive elements (``fields_from_words``) and a call serves
sixteen, i.e. one quantization block.  Elements 0 and 1 of a group share the
word's bytes 2 and 0 (element 1 reads them bit-reversed), elements 2 and 3
bytes 3 and 1: this is how the sm_100a conversion with random bits
(cvt.rs ... e2m1x4) consumes its 32-bit operand, so the device converts a
group in one instruction.  Each element's 16 bits are uniform; the two
elements sharing bytes see them with the bit order reversed.

Pins (tests/test_oracle_philox.py): the published known-answer vectors of
Philox4x32-10, plus uniformity checks of the derived streams.
"""

import numpy as np

M0 = np.uint64(0xD2511F53)
M1 = np.uint64(0xCD9E8D57)
W0 = 0x9E3779B9
W1 = 0xBB67AE85
MASK32 = np.uint64(0xFFFFFFFF)
SHIFT32 = np.uint64(32)

PURPOSE_SAMPLE = 1
PURPOSE_OMEGA = 2
PURPOSE_SR = 3

SR_SUB_ROWWISE = 0   # residual, 16-blocks along columns
SR_SUB_COLWISE = 1   # residual, 16-blocks along rows
SR_SUB_LEFT = 2      # left factor (U), blocks along its rows
SR_SUB_RIGHT = 3     # right factor (V), blocks along its rows


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox rounds on (vectors of) 32-bit counters; returns 4 word arrays."""
    c0 = np.asarray(c0, dtype=np.uint64) & MASK32
    c1 = np.asarray(c1, dtype=np.uint64) & MASK32
    c2 = np.asarray(c2, dtype=np.uint64) & MASK32
    c3 = np.asarray(c3, dtype=np.uint64) & MASK32
    k0 = int(k0) & 0xFFFFFFFF
    k1 = int(k1) & 0xFFFFFFFF
    for r in range(10):
        if r > 0:
            k0 = (k0 + W0) & 0xFFFFFFFF
            k1 = (k1 + W1) & 0xFFFFFFFF
        p0 = M0 * c0          # < 2^64, exact in uint64
        p1 = M1 * c2
        hi0, lo0 = p0 >> SHIFT32, p0 & MASK32
        hi1, lo1 = p1 >> SHIFT32, p1 & MASK32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(k0), lo1,
                          hi0 ^ c3 ^ np.uint64(k1), lo0)
    return c0, c1, c2, c3


def tag(operand_id, purpose, sub=0):
    return ((int(operand_id) & 0xFFFFFF) << 8) | ((purpose & 0xF) << 4) | (sub & 0xF)


def stream_words(seed, tag_value, step, q):
    """The four words of counters ``q`` (uint64 array) -> uint64 array (len(q), 4)."""
    q = np.asarray(q, dtype=np.uint64)
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    w = philox4x32_10(q & MASK32, q >> SHIFT32,
                      np.full(q.shape, tag_value, dtype=np.uint64),
                      np.full(q.shape, int(step) & 0xFFFFFFFF, dtype=np.uint64),
                      seed & 0xFFFFFFFF, seed >> 32)
    return np.stack(w, axis=-1)


def element_words(seed, tag_value, step, n):
    """Word ``e & 3`` of counter ``e >> 2`` for elements e = 0..n-1 (uint64)."""
    q = np.arange((n + 3) // 4, dtype=np.uint64)
    return stream_words(seed, tag_value, step, q).reshape(-1)[:n]


def _rev16(x):
    """Bit reversal of 16-bit values (bit 0 <-> bit 15)."""
    x = np.asarray(x, dtype=np.uint64)
    r = np.zeros_like(x)
    for b in range(16):
        r |= ((x >> np.uint64(b)) & np.uint64(1)) << np.uint64(15 - b)
    return r


def fields_from_words(words, position):
    """16-bit rounding field of the element at ``position`` (0..3) of a 4-group.

    One 32-bit word W (bytes b0 = bits 0-7 .. b3 = bits 24-31) rounds four
    consecutive elements: positions 0 and 1 take the 16 bits b2:b0 (b2 high),
    position 0 as they are and position 1 bit-reversed; positions 2 and 3 take
    b3:b1 the same way.
    """
    w = np.asarray(words, dtype=np.uint64)
    pos = np.asarray(position, dtype=np.uint64)
    byte = [(w >> np.uint64(8 * t)) & np.uint64(0xFF) for t in range(4)]
    f02 = (byte[2] << np.uint64(8)) | byte[0]
    f13 = (byte[3] << np.uint64(8)) | byte[1]
    base = np.where(pos < 2, f02, f13)
    return np.where((pos & np.uint64(1)) == 1, _rev16(base), base).astype(np.int64)


def sr_fields(seed, operand_id, sub, step, n):
    """16-bit stochastic-rounding fields for elements e = 0..n-1 (int64 in [0, 65535]).

    Element e is at position ``e & 3`` of the 4-group served by word
    ``(e >> 2) & 3`` of counter ``e >> 4``: one call serves sixteen consecutive
    elements, i.e. exactly one 16-element quantization block.
    """
    e = np.arange(n, dtype=np.uint64)
    return sr_fields_at(seed, operand_id, sub, step, e)


def sr_fields_at(seed, operand_id, sub, step, elements):
    """The same fields as ``sr_fields`` for arbitrary element indices."""
    e = np.asarray(elements, dtype=np.uint64)
    q = e >> np.uint64(4)
    uq, inv = np.unique(q, return_inverse=True)
    words = stream_words(seed, tag(operand_id, PURPOSE_SR, sub), step, uq)
    w = words[inv.reshape(-1), ((e.reshape(-1) >> np.uint64(2)) & np.uint64(3)).astype(np.int64)]
    return fields_from_words(w, (e.reshape(-1) & np.uint64(3))).reshape(e.shape)
