"""The word-wide XOR identities the CUDA decoder uses, checked against the oracle on the CPU.

The kernels decode a 32-weight block with shifted XORs of its two bit planes instead of walking
the state weight by weight. This test restates those identities in numpy (test-only code; the
kernels are CUDA) and compares them with the oracle's step-by-step decoder for every 16-bit state
and for random multi-block rows, with and without a carry from the previous block. The GPU
parity tests then check the kernels themselves bit for bit.
"""
import os
import re

import numpy as np

import oracle
from trellis_coded_fp4_b200 import synth

M32 = np.uint64(0xFFFFFFFF)


def _dly(x, px, d):
    return ((x << np.uint64(d)) | (px >> np.uint64(32 - d))) & M32


def _planes(L, H, pL, pH):
    L, H, pL, pH = (np.asarray(v, np.uint64) for v in (L, H, pL, pH))
    Ld = {d: _dly(L, pL, d) for d in range(1, 8)}
    Hd = {d: _dly(H, pH, d) for d in range(1, 8)}
    neg = ~(H ^ Ld[7] ^ Ld[4] ^ Ld[2] ^ Hd[1]) & M32
    n0 = neg ^ Ld[7] ^ Hd[6] ^ Hd[4] ^ Ld[1]
    n1 = neg ^ Hd[7] ^ Ld[5] ^ Ld[3] ^ Hd[1]
    n2 = neg ^ L ^ Ld[6] ^ Hd[5] ^ Hd[3] ^ Hd[2]
    return n0, n1, n2, neg


def _codes_from_planes(n):
    i = np.arange(32, dtype=np.uint64)
    return sum(((n[c][..., None] >> i) & np.uint64(1)) << np.uint64(c) for c in range(4)).astype(np.uint8)


def test_identity_for_every_state():
    # The last weight of a block decoded after a 7-symbol history covers every 16-bit state.
    s = np.arange(1 << 16, dtype=np.uint64)
    # state bits 2m / 2m+1 hold symbol i-7+m; place history in the previous block's top bits and
    # the current symbol at bit 0 of this block, then read weight 0's code.
    pL = np.zeros_like(s)
    pH = np.zeros_like(s)
    for m in range(7):
        pL |= ((s >> np.uint64(2 * m)) & np.uint64(1)) << np.uint64(25 + m)
        pH |= ((s >> np.uint64(2 * m + 1)) & np.uint64(1)) << np.uint64(25 + m)
    L = (s >> np.uint64(14)) & np.uint64(1)
    H = (s >> np.uint64(15)) & np.uint64(1)
    codes = _codes_from_planes(_planes(L, H, pL, pH))[:, 0]
    ref = np.array([oracle.state_code(int(v)) for v in s], np.uint8)
    assert (codes == ref).all()


def test_identity_on_rows_with_and_without_carry():
    rows, cols = 8, 256
    st = synth.stream(rows, cols, seed=51).astype(np.uint64)
    for seg_len in (32, 128, 256):
        ref = oracle.decode_codes(st.astype(np.uint32), rows, cols, seg_len)
        sb = seg_len // 32
        got = np.zeros((rows, cols), np.uint8)
        for j in range(cols // 32):
            L, H = st[:, j, 0], st[:, j, 1]
            if j % sb == 0:
                pL = pH = np.zeros(rows, np.uint64)
            else:
                pL, pH = st[:, j - 1, 0], st[:, j - 1, 1]
            got[:, 32 * j:32 * j + 32] = _codes_from_planes(_planes(L, H, pL, pH))
        assert (got == ref).all(), seg_len


# ----------------------------------------------------------------------------- nibble transposes
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "trellis_coded_fp4_b200", "csrc", "tcf4_device.cuh")


def _lop3(a, b, c, lut):
    """Bitwise three-input function by truth table: bit (a<<2 | b<<1 | c) of lut."""
    out = np.zeros_like(a)
    for i in range(8):
        if (lut >> i) & 1:
            ma = a if i & 4 else ~a
            mb = b if i & 2 else ~b
            mc = c if i & 1 else ~c
            out |= ma & mb & mc
    return out & M32


def _luts(fn_name, next_name):
    text = open(HEADER).read()
    body = text[text.index("void " + fn_name + "("):text.index(next_name)]
    return [int(v, 16) for v in re.findall(r"lop3\.b32 %0, %1, %2, %3, (0x[0-9A-Fa-f]+);", body)]


def test_delta_swap_select_table():
    # Each three-input op in delta_swap takes operands (x, y, mask) and must compute mask ? x : y;
    # delta_swap_inv_b reads its second word inverted: mask ? x : ~y, then mask ? ~x : y.
    rng = np.random.default_rng(7)
    x, y, m = (rng.integers(0, 1 << 32, 64, dtype=np.uint64) for _ in range(3))
    sel = lambda m, x, y: ((m & x) | (~m & y)) & M32  # noqa: E731
    luts = _luts("delta_swap", "delta_swap_inv_b")
    assert len(luts) == 2
    for lut in luts:
        assert (_lop3(x, y, m, lut) == sel(m, x, y)).all(), hex(lut)
    inv = _luts("delta_swap_inv_b", "void planes_to_nibbles_interleaved")
    assert len(inv) == 2
    assert (_lop3(x, y, m, inv[0]) == sel(m, x, ~y & M32)).all(), hex(inv[0])
    assert (_lop3(x, y, m, inv[1]) == sel(m, ~x & M32, y)).all(), hex(inv[1])


def test_transpose_absorbing_the_inversion():
    # planes_to_nibbles_interleaved_i3 (n3 given inverted, swaps emulated with the header's LUTs)
    # equals the plain transpose of the true planes
    luts, inv = _luts("delta_swap", "delta_swap_inv_b"), _luts("delta_swap_inv_b", "void planes_to_nibbles_interleaved")
    rng = np.random.default_rng(10)
    n = [rng.integers(0, 1 << 32, 256, dtype=np.uint64) for _ in range(4)]

    def swap(a, b, s, mask, l0, l1):
        ms = np.uint64(mask)
        nb = _lop3(a >> np.uint64(s), b, ms, l0)
        na = _lop3((b << np.uint64(s)) & M32, a, (ms << np.uint64(s)) & M32, l1)
        return na, nb
    a, b = swap(n[0], n[1], 1, 0x55555555, *luts)
    c, d = swap(n[2], ~n[3] & M32, 1, 0x55555555, *inv)
    a, c = swap(a, c, 2, 0x33333333, *luts)
    b, d = swap(b, d, 2, 0x33333333, *luts)
    ra, rb = _delta_swap(n[0], n[1], 1, 0x55555555)
    rc, rd = _delta_swap(n[2], n[3], 1, 0x55555555)
    ra, rc = _delta_swap(ra, rc, 2, 0x33333333)
    rb, rd = _delta_swap(rb, rd, 2, 0x33333333)
    for got, ref in zip((a, b, c, d), (ra, rb, rc, rd)):
        assert (got == ref).all()


def _delta_swap(a, b, s, mask):
    mask = np.uint64(mask)
    nb = (mask & (a >> np.uint64(s))) | (~mask & b & M32)
    ms = (mask << np.uint64(s)) & M32
    na = (ms & (b << np.uint64(s)) & M32) | (~ms & a & M32)
    return na, nb


def test_interleaved_nibble_order():
    # planes -> four words with weight 4v+j in nibble v of word j (the order the MMA operands use)
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 16, (16, 32)).astype(np.uint64)
    n = [sum(((codes[:, i] >> np.uint64(c)) & np.uint64(1)) << np.uint64(i) for i in range(32)) for c in range(4)]
    a, b = _delta_swap(n[0], n[1], 1, 0x55555555)
    c, d = _delta_swap(n[2], n[3], 1, 0x55555555)
    a, c = _delta_swap(a, c, 2, 0x33333333)
    b, d = _delta_swap(b, d, 2, 0x33333333)
    for j, w in enumerate((a, b, c, d)):
        for v in range(8):
            assert ((w >> np.uint64(4 * v)) & np.uint64(15) == codes[:, 4 * v + j]).all()


def test_factored_segment_start_form():
    # The segment-start decoder shifts shared XOR sums once (F = L ^ L<<2, U = L ^ L<<6,
    # G = H ^ H<<2); restated here, it must equal the term-by-term planes for random blocks.
    rng = np.random.default_rng(9)
    L = rng.integers(0, 1 << 32, 4096, dtype=np.uint64)
    H = rng.integers(0, 1 << 32, 4096, dtype=np.uint64)
    z = np.zeros_like(L)
    ref = _planes(L, H, z, z)

    def s(x, d):
        return (x << np.uint64(d)) & M32
    F, U, H2 = L ^ s(L, 2), L ^ s(L, 6), s(H, 2)
    G = H ^ H2
    X = H ^ s(F, 2) ^ s(L, 7)
    q1h = X ^ s(H, 1)
    got = ((~(q1h ^ s(U, 1) ^ s(G, 4))) & M32, (~(X ^ s(F, 3) ^ s(H, 7))) & M32,
           (~(q1h ^ U ^ s(G, 3) ^ H2)) & M32, (~q1h) & M32)
    for a, b in zip(got, ref):
        assert (a == b).all()


def _decoder_luts(fn_name, next_name):
    """The lop3<...> truth tables of a decoder in the header, in source order."""
    text = open(HEADER).read()
    body = text[text.index("Planes " + fn_name + "("):text.index(next_name)]
    return [int(v, 16) for v in re.findall(r"lop3<(0x[0-9A-Fa-f]+)>\(", body)]


def test_decoder_truth_tables_match_the_identity():
    # The decoders write their XOR sums as three-input ops with immediate truth tables. Applied in
    # the header's source order to the same operands, those tables must give the planes of the
    # identity above (checked against the oracle for every state), with and without a carry.
    rng = np.random.default_rng(11)
    L, H, pL, pH = (rng.integers(0, 1 << 32, 512, dtype=np.uint64) for _ in range(4))
    t = _decoder_luts("decode_block", "// Segment-start form")
    assert len(t) == 9
    Ld = {d: _dly(L, pL, d) for d in range(1, 8)}
    Hd = {d: _dly(H, pH, d) for d in range(1, 8)}
    neg = _lop3(H, _lop3(Ld[7], Ld[4], Ld[2], t[1]), Hd[1], t[0])
    n0 = _lop3(neg, _lop3(Ld[7], Hd[6], Hd[4], t[3]), Ld[1], t[2])
    n1 = _lop3(neg, _lop3(Hd[7], Ld[5], Ld[3], t[5]), Hd[1], t[4])
    n2 = _lop3(_lop3(neg, L, Ld[6], t[7]), _lop3(Hd[5], Hd[3], np.zeros_like(L), t[8]), Hd[2], t[6])
    for got, ref in zip((n0, n1, n2, neg), _planes(L, H, pL, pH)):
        assert (got == ref).all()
    # segment-start form, n3 returned inverted
    t = _decoder_luts("decode_block0_i3", "__device__ __forceinline__ Planes decode_block0(")
    assert len(t) == 9
    z = np.zeros_like(L)
    sh = lambda x, d: (x << np.uint64(d)) & M32  # noqa: E731
    F, U, H2 = _lop3(L, sh(L, 2), z, t[0]), _lop3(L, sh(L, 6), z, t[1]), sh(H, 2)
    tt = _lop3(U, sh(_lop3(H, H2, z, t[3]), 3), z, t[2])
    X = _lop3(H, sh(F, 2), sh(L, 7), t[4])
    q1h = _lop3(X, sh(H, 1), z, t[5])
    n0 = _lop3(q1h, sh(tt, 1), z, t[6])
    n1 = _lop3(X, sh(F, 3), sh(H, 7), t[7])
    n2 = _lop3(q1h, tt, H2, t[8])
    for got, ref in zip((n0, n1, n2, ~q1h & M32), _planes(L, H, z, z)):
        assert (got == ref).all()
