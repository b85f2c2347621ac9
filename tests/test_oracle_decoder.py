"""Pins for the oracle's XOR-Trellis decoder and MXFP4 expansion (CPU only).

Each test checks the oracle against something other than itself: the constants the pages print
(tests/golden), the E2M1 definition, and the structural properties the pages state for the
decoder (one palette per state, 15 distinct E2M1 values, uniform use of the palettes).
"""
import os

import numpy as np
import pytest

import oracle
from trellis_coded_fp4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def test_tables_match_printed_constants():
    g = _read_golden("xor_trellis_constants.txt")
    pal, masks = oracle.tables()
    for p in range(4):
        printed = [float(v) for v in g[f"P{p}"]]
        assert list(pal[p]) == printed, f"palette P{p}"
    assert [int(m, 16) for m in g["masks"]] == [int(m) for m in masks]


def test_masks_cover_exactly_the_predecessor_window():
    # The reading "new symbol enters at bits 14-15" rests on this: the union of the printed
    # masks is bits 0..13, so parities never see the branch being decoded.
    g = _read_golden("xor_trellis_constants.txt")
    masks = [int(m, 16) for m in g["masks"]]
    union = 0
    for m in masks:
        union |= m
    assert union == 0x3FFF
    # GF(2) rank 4: the four parities are independent linear functions of the window.
    rows = list(masks)
    rank = 0
    for bit in range(16):
        piv = next((r for r in rows if (r >> bit) & 1), None)
        if piv is None:
            continue
        rows.remove(piv)
        rows = [r ^ piv if (r >> bit) & 1 else r for r in rows]
        rank += 1
    assert rank == 4


def test_e2m1_value_definition():
    g = _read_golden("mxfp4_definitions.txt")
    doubled = [int(v) for v in g["doubled_magnitudes"]]
    mags = [oracle.e2m1_value(c) for c in range(8)]
    assert [2 * m for m in mags] == doubled          # codes 0..7 in increasing order
    for c in range(8):
        neg = oracle.e2m1_value(c | 8)
        assert neg == -mags[c] and np.signbit(neg)   # sign bit 3 negates, including -0
    assert oracle.ue8m0_value(127) == 1.0 and oracle.ue8m0_value(120) == 2.0 ** -7
    assert np.isnan(oracle.ue8m0_value(255))


def _all_windows():
    return range(1 << 14)


def test_every_state_maps_its_four_branches_into_one_palette():
    # Decoder bullet: (p0, p1) select the palette, (q0, q1) permute branch -> entry. Under the
    # chosen shift reading the four branches of every predecessor window must use one palette
    # and four distinct entries. A push at the low end (or a wrong mask) breaks this.
    for w in _all_windows():
        ps, es = set(), set()
        for b in range(4):
            p, e = oracle.state_decode(w | (b << 14))
            ps.add(p)
            es.add(e)
        assert len(ps) == 1 and es == {0, 1, 2, 3}, hex(w)


def test_values_are_e2m1_and_cover_the_15_values():
    g = _read_golden("mxfp4_definitions.txt")
    e2m1 = {oracle.e2m1_value(c) for c in range(16)}
    seen = set()
    for s in range(1 << 16):
        v = oracle.state_value(s)
        assert v in e2m1
        seen.add(v)
    assert len(seen) == int(g["distinct_values"][0]) == len(e2m1)


def test_uniform_use_of_palettes_and_permutations():
    counts = np.zeros((4, 4), int)
    for w in _all_windows():
        p, q = oracle.state_decode(w)        # branch 0: entry e = 0 xor q = q
        counts[p, q] += 1
    assert (counts == 1024).all()


def test_state_code_is_the_e2m1_encoding_of_the_value():
    codes = set()
    for s in range(1 << 16):
        c = oracle.state_code(s)
        v = oracle.state_value(s)
        assert c < 16
        cv = oracle.e2m1_value(c)
        assert cv == v and np.signbit(cv) == np.signbit(v)
        codes.add(c)
    assert codes == set(range(16))           # the 16 palette slots are the 16 codes


def test_state_push_is_a_sliding_window():
    # After pushing b_0..b_7 the 16-bit state holds b_m at bits 2m..2m+1 (oldest lowest);
    # built here from the little-endian integer of the interleaved bit string.
    r = np.random.default_rng(1)
    for _ in range(200):
        syms = r.integers(0, 4, 12)
        s = 0
        for b in syms:
            s = oracle.state_push(s, int(b))
        bitstring = "".join(format(int(b), "02b")[::-1] for b in syms[-8:])  # LSB-first pairs
        assert s == int(bitstring[::-1], 2)


def _scalar_decode(stream, rows, cols, seg_len):
    """Per-weight decode through the scalar entry points, for the bulk functions."""
    codes = np.zeros((rows, cols), np.uint8)
    for n in range(rows):
        s = 0
        for k in range(cols):
            if k % seg_len == 0:
                s = 0
            lo, hi = stream[n, k // 32]
            b = ((int(lo) >> (k % 32)) & 1) | (((int(hi) >> (k % 32)) & 1) << 1)
            s = oracle.state_push(s, b)
            codes[n, k] = oracle.state_code(s)
    return codes


@pytest.mark.parametrize("seg_len", [32, 64, 128])
def test_bulk_decode_matches_scalar_steps(seg_len):
    rows, cols = 3, 128
    st = synth.stream(rows, cols, seed=11)
    assert (oracle.decode_codes(st, rows, cols, seg_len) == _scalar_decode(st, rows, cols, seg_len)).all()


def test_segments_restart_from_state_zero():
    rows, cols = 4, 256
    st = synth.stream(rows, cols, seed=12)
    full = oracle.decode_codes(st, rows, cols, 32)
    for j in range(cols // 32):                 # each 32-block decodes on its own
        one = oracle.decode_codes(st[:, j:j + 1].copy(), rows, 32, 32)
        assert (one == full[:, 32 * j:32 * j + 32]).all()
    long = oracle.decode_codes(st, rows, cols, cols)
    assert (long[:, :32] == full[:, :32]).all()  # first block: same initial state
    assert (long[:, 32:] != full[:, 32:]).any()  # later blocks carry the window across blocks


def test_expansion_packs_codes_and_copies_scales():
    rows, cols = 5, 96
    st = synth.stream(rows, cols, seed=13)
    sc = synth.scales(rows, cols, seed=13)
    for seg_len in (32, 96):
        nib, osc = oracle.expand_mxfp4(st, sc, rows, cols, seg_len)
        codes = oracle.decode_codes(st, rows, cols, seg_len)
        assert (nib & 0xF == codes[:, 0::2]).all() and (nib >> 4 == codes[:, 1::2]).all()
        assert (osc == sc).all()
        # MXFP4 dequantisation of the expanded tensor equals the decoded weights.
        w = oracle.decode_values(st, sc, rows, cols, seg_len)
        deq = np.array([[oracle.e2m1_value(c) for c in row] for row in codes])
        deq *= np.repeat(2.0 ** (sc.astype(np.float64) - 127), 32, axis=1)
        assert (deq == w).all()
