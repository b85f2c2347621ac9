"""Pins for the oracle's interleaved packing: its sliding-window decode and its repack to planar.

The XOR-Trellis news page's "XOR-Trellis FP4 decoder" bullet keys each weight on a 16-bit sliding
state. Under the interleaved packing (one bit string per row, two bits per symbol, low bit first)
that state is a 16-bit window of the string itself. The oracle decodes such a stream that way, with
no symbol recurrence, and separately repacks it to the planar words the recurrence decoder reads.
The two routes share nothing but the state -> code step, so their agreement pins the repack's bit
mapping (a swapped plane, a swapped word or an off-by-one window fails it).
"""
import numpy as np
import pytest

import oracle


def _random_il(rows, cols, seed):
    return np.random.default_rng(seed).integers(0, 2**32, size=(rows, cols // 32, 2), dtype=np.uint32)


@pytest.mark.parametrize("cols,seg", [(64, 32), (128, 64), (96, 96), (256, 128)])
def test_window_decode_equals_recurrence_decode_of_the_repack(cols, seg):
    rows = 3
    il = _random_il(rows, cols, 100 + cols + seg)
    direct = oracle.decode_codes_interleaved(il, rows, cols, seg)
    planar = oracle.repack_interleaved(il, rows, cols)
    assert np.array_equal(direct, oracle.decode_codes(planar, rows, cols, seg))


def test_single_symbols_by_hand():
    # symbol 5 = 3: string bits 10 and 11 (word 0) -> bit 5 of both planes
    il = np.zeros((1, 1, 2), np.uint32)
    il[0, 0, 0] = 0xC00
    assert oracle.repack_interleaved(il, 1, 32).tolist() == [[[1 << 5, 1 << 5]]]
    # symbol 18 = 2 (high bit only): string bit 37 = bit 5 of word 1 -> bit 18 of the high plane
    il[0, 0, 0], il[0, 0, 1] = 0, 1 << 5
    assert oracle.repack_interleaved(il, 1, 32).tolist() == [[[0, 1 << 18]]]
    # second block of a row: symbol 32 = 1 -> string bit 64 = bit 0 of the row's word 2
    il = np.zeros((1, 2, 2), np.uint32)
    il[0, 1, 0] = 1
    assert oracle.repack_interleaved(il, 1, 64).tolist() == [[[0, 0], [1, 0]]]


def test_uniform_strings():
    il = np.full((2, 2, 2), 0x55555555, np.uint32)  # every symbol = 1
    assert np.array_equal(oracle.repack_interleaved(il, 2, 64), np.tile(np.array([0xFFFFFFFF, 0], np.uint32), (2, 2, 1)))
    il = np.full((2, 2, 2), 0xAAAAAAAA, np.uint32)  # every symbol = 2
    assert np.array_equal(oracle.repack_interleaved(il, 2, 64), np.tile(np.array([0, 0xFFFFFFFF], np.uint32), (2, 2, 1)))


def test_repack_is_a_bit_permutation():
    # each of the 64 single-bit strings of a block maps to a single bit, and no two to the same one
    seen = set()
    for p in range(64):
        il = np.zeros((1, 1, 2), np.uint32)
        il[0, 0, p // 32] = 1 << (p % 32)
        out = oracle.repack_interleaved(il, 1, 32).reshape(-1)
        bits = [(w, b) for w in range(2) for b in range(32) if (int(out[w]) >> b) & 1]
        assert len(bits) == 1
        seen.add(bits[0])
    assert len(seen) == 64


def test_window_sees_zeros_before_the_segment_start():
    # all-ones string, segments of 32: the first weight of each segment has state 0xC000 (only its
    # own symbol), the eighth and later have the full window 0xFFFF
    rows, cols, seg = 1, 64, 32
    il = np.full((rows, cols // 32, 2), 0xFFFFFFFF, np.uint32)
    codes = oracle.decode_codes_interleaved(il, rows, cols, seg)
    for k0 in (0, 32):
        assert codes[0, k0] == oracle.state_code(0xC000)
        assert codes[0, k0 + 1] == oracle.state_code(0xF000)
        assert all(codes[0, k0 + i] == oracle.state_code(0xFFFF) for i in range(7, 32))


def test_shape_errors():
    il = np.zeros((1, 1, 2), np.uint32)
    with pytest.raises(Exception):
        oracle.decode_codes_interleaved(il, 1, 32, 48)
