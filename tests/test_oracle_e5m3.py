"""Pins for the oracle's E5M3 block-scale variant (CPU only).

The XOR-Trellis news page names E5M3 block scales without an encoding; the reading is stated in
tests/golden/e5m3_reading.txt. Pinned here: the hand-worked values of that fixture, monotonicity
and even spacing within each binade, the reduction to the UE8M0 path when the mantissa is zero,
and exact rational products.
"""
import os
from fractions import Fraction

import numpy as np

import oracle
from trellis_coded_fp4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e5m3_reading.txt")


def _fixture():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            b, v = line.split()
            rows.append((int(b, 16), v))
    return rows


def test_hand_worked_values():
    for b, v in _fixture():
        got = oracle.e5m3_value(b)
        if v == "nan":
            assert np.isnan(got), hex(b)
        else:
            assert Fraction(got) == Fraction(v), hex(b)


def test_every_finite_byte_is_increasing_and_evenly_spaced_per_binade():
    vals = [oracle.e5m3_value(b) for b in range(0xF8)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    assert all(np.isnan(oracle.e5m3_value(b)) for b in range(0xF8, 0x100))
    for e in range(1, 31):  # eight values per binade, step 2^(e-15)/8; subnormals step 2^-17
        step = [vals[8 * e + m + 1] - vals[8 * e + m] for m in range(7)]
        assert all(s == 2.0 ** (e - 18) for s in step)
    assert all(vals[m + 1] - vals[m] == 2.0 ** -17 for m in range(8))


def test_zero_mantissa_reduces_to_ue8m0():
    rows, cols = 3, 96
    st = synth.stream(rows, cols, 31)
    e = np.random.default_rng(31).integers(1, 31, (rows, cols // 32)).astype(np.uint8)
    w5 = oracle.decode_values(st, (e << 3).astype(np.uint8), rows, cols, 32, scale_fmt="e5m3")
    w8 = oracle.decode_values(st, (e + 112).astype(np.uint8), rows, cols, 32)
    assert np.array_equal(w5, w8)


def test_e5m3_gemv_equals_exact_rational_sum():
    rows, cols, T = 3, 64, 2
    st = synth.stream(rows, cols, 32)
    sc = np.random.default_rng(32).integers(0x60, 0x90, (rows, cols // 32)).astype(np.uint8)
    xb = synth.bf16_bits(synth.activations(T, cols, 32))
    for seg in (32, 64):
        y, wn = oracle.gemv(st, sc, rows, cols, seg, xb, scale_fmt="e5m3")
        codes = oracle.decode_codes(st, rows, cols, seg)
        x = oracle.bf16_bits_to_f64(xb)
        for n in range(rows):
            w = [Fraction(oracle.e2m1_value(int(codes[n, k]))) * Fraction(oracle.e5m3_value(int(sc[n, k // 32])))
                 for k in range(cols)]
            assert abs(float(wn[n]) - float(np.sqrt(float(sum(v * v for v in w))))) <= 1e-12 * float(wn[n])
            for t in range(T):
                exact = sum(a * Fraction(float(b)) for a, b in zip(w, x[t]))
                bound = cols * 2.0 ** -53 * float(sum(abs(a) * abs(Fraction(float(b))) for a, b in zip(w, x[t])))
                assert abs(Fraction(y[t, n]) - exact) <= Fraction(bound)
