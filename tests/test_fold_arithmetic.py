"""The byte arithmetic that folds an integer scale into the unpacked weight
operand, checked exhaustively on the CPU.

The tile kernel turns four offset codes u_i = q_i + 8 (one per byte of a
32-bit word) into the int8 bytes S * q_i with one multiply-add and one XOR:
bytes of ((word * S + (128 - 8 S) * 0x01010101) mod 2^32) ^ 0x80808080.  The
claim is that this is exact whenever every S * q_i lies in [-128, 127] (so for
every code when 0 <= S <= 16, and for S = 17 or 18 when no code is -8), and
that it fails outside that range, which is why the kernel checks the range
before folding.  Here every word of four codes is tried for every such S."""
import itertools

import numpy as np


def _folded_bytes(codes, S):
    """codes: int array [..., 4] in [-8, 7]; returns the 4 result bytes as int8."""
    u = (codes.astype(np.int64) + 8).astype(np.uint64)
    word = u[..., 0] | (u[..., 1] << 8) | (u[..., 2] << 16) | (u[..., 3] << 24)
    k1 = ((128 - 8 * S) * 0x01010101) % (1 << 32)
    r = (word * np.uint64(S) + np.uint64(k1)) % np.uint64(1 << 32)
    r ^= np.uint64(0x80808080)
    out = np.stack([(r >> np.uint64(8 * i)) & np.uint64(0xFF) for i in range(4)], axis=-1)
    return out.astype(np.uint8).view(np.int8)


def _all_words(qmin):
    vals = np.arange(qmin, 8)
    return np.array(list(itertools.product(vals, repeat=4)), np.int64)


def test_exact_for_every_code_up_to_16():
    words = _all_words(-8)
    for S in range(0, 17):
        assert np.array_equal(_folded_bytes(words, S).astype(np.int64), S * words), S


def test_exact_for_17_and_18_without_the_code_minus_8():
    words = _all_words(-7)
    for S in (17, 18):
        assert np.array_equal(_folded_bytes(words, S).astype(np.int64), S * words), S


def test_not_exact_outside_the_int8_range():
    # S = 17 with the code -8, and S = 19 with the code 7, leave int8: the
    # kernel must not fold them
    w = np.array([[-8, 0, 0, 0], [7, 1, 2, 3]], np.int64)
    assert not np.array_equal(_folded_bytes(w[:1], 17).astype(np.int64), 17 * w[:1])
    assert not np.array_equal(_folded_bytes(w[1:], 19).astype(np.int64), 19 * w[1:])


def test_code_minus_8_detector():
    """The scan's test for the code -8 (nibble 1000) in a word of packed
    codes: bit 3 set and bits 0-2 clear, found without a carry between
    nibbles.  Every combination of four nibbles, in either half of the word."""
    w = np.arange(1 << 16, dtype=np.uint64)
    for shift in (0, 16):
        x = (w << np.uint64(shift)) % np.uint64(1 << 32)
        low_nonzero = ((x & np.uint64(0x77777777)) + np.uint64(0x77777777)) & np.uint64(0x88888888)
        found = (x & np.uint64(0x88888888) & ~low_nonzero & np.uint64(0xFFFFFFFF)) != 0
        nibbles = np.stack([(w >> np.uint64(4 * i)) & np.uint64(0xF) for i in range(4)], axis=-1)
        assert np.array_equal(found, (nibbles == 8).any(axis=-1))
