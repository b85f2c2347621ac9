"""Pins for the oracle's products from a resident MXFP4 tensor (HEPH serving mode 2, consumer side).

The MXFP4 element is E2M1(code) * 2^(E-127) (OCP MX, "Tied Trit-Planes" section 2.1); the E2M1
magnitudes here come from the doubled integers printed in section 2.3 (tests/golden), not from the
oracle's formula. Pins: exact rational sums, one-hot activations selecting single elements (which
fixes the nibble order and the scale index), and the identity "expand, then multiply" equals the
fused trellis product exactly (both are fp64 sums of the same exact products in the same order).
"""
import dataclasses
import os
from fractions import Fraction

import numpy as np

import oracle
from trellis_coded_fp4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_definitions.txt")


def _doubled_magnitudes():
    for line in open(GOLDEN):
        if line.startswith("doubled_magnitudes"):
            return [int(v) for v in line.split()[1:]]
    raise AssertionError("doubled_magnitudes missing from the golden file")


def _element(code, E):
    """Exact value of an MXFP4 element: sign bit 3, magnitude index = low 3 bits."""
    mag = Fraction(_doubled_magnitudes()[code & 7], 2)
    v = -mag if code & 8 else mag
    return v * (Fraction(2) ** (E - 127))


def _random_mx(rows, cols, seed, lo=118, hi=130):
    rng = np.random.default_rng(seed)
    nib = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    sc = rng.integers(lo, hi, size=(rows, cols // 32), dtype=np.uint8)
    return nib, sc


def test_mxfp4_gemv_equals_exact_rational_sum():
    rows, cols, T = 3, 96, 2
    nib, sc = _random_mx(rows, cols, 5)
    xb = synth.bf16_bits(synth.activations(T, cols, 5))
    y, wn = oracle.mxfp4_gemv(nib, sc, rows, cols, xb)
    x = oracle.bf16_bits_to_f64(xb)
    for n in range(rows):
        w = [_element((int(nib[n, k // 2]) >> (4 * (k % 2))) & 15, int(sc[n, k // 32])) for k in range(cols)]
        assert abs(float(sum(v * v for v in w)) ** 0.5 - wn[n]) <= 1e-12 * wn[n]
        for t in range(T):
            exact = sum(v * Fraction(float(x[t, k])) for k, v in enumerate(w))
            bound = cols * 2.0 ** -53 * sum(abs(float(v)) * abs(float(x[t, k])) for k, v in enumerate(w))
            assert abs(Fraction(y[t, n]) - exact) <= Fraction(bound)


def test_mxfp4_gemv_one_hot_selects_elements():
    rows, cols = 2, 64
    nib, sc = _random_mx(rows, cols, 6)
    for k in (0, 1, 31, 32, 33, 63):           # low and high nibbles, both scale blocks
        x = np.zeros((1, cols), np.uint16)
        x[0, k] = 0x3F80                          # bf16 1.0
        y, _ = oracle.mxfp4_gemv(nib, sc, rows, cols, x)
        for n in range(rows):
            code = (int(nib[n, k // 2]) >> (4 * (k % 2))) & 15
            assert Fraction(y[0, n]) == _element(code, int(sc[n, k // 32]))


def test_mxfp4_gemv_of_expansion_equals_fused_product():
    rows, cols, T = 7, 192, 3
    for seg_len in (32, 192):
        st = synth.stream(rows, cols, 8)
        sc = synth.scales(rows, cols, 8)
        xb = synth.bf16_bits(synth.activations(T, cols, 8))
        nib, sc2 = oracle.expand_mxfp4(st, sc, rows, cols, seg_len)
        y1, w1 = oracle.gemv(st, sc, rows, cols, seg_len, xb)
        y2, w2 = oracle.mxfp4_gemv(nib, sc2, rows, cols, xb, row_ids=None)
        assert np.array_equal(y1, y2) and np.array_equal(w1, w2)
        y3, _ = oracle.mxfp4_gemv(nib, sc2, rows, cols, xb, row_ids=[6, 0, 3])
        assert np.array_equal(y3, y1[:, [6, 0, 3]])


def test_moe_on_expanded_experts_equals_fused_layer():
    E, H, I = 3, 64, 96
    layer = synth.moe_layer(E, H, I, seed=9)
    xb = synth.bf16_bits(synth.activations(2, H, seed=9))
    ids = np.array([[2, 0], [1, 2]], np.int32)
    w = np.array([[0.75, 0.25], [0.5, 0.5]])
    out1, h1 = oracle.moe(layer, xb, ids, w, 32)
    gun, gus, dnn, dns = [], [], [], []
    for e in range(E):
        a, b = oracle.expand_mxfp4(layer.gu_stream[e], layer.gu_scales[e], 2 * I, H, 32)
        c, d = oracle.expand_mxfp4(layer.dn_stream[e], layer.dn_scales[e], H, I, 32)
        gun.append(a), gus.append(b), dnn.append(c), dns.append(d)

    @dataclasses.dataclass
    class MxLayer:
        E: int
        H: int
        I: int
        gu_nibbles: list
        gu_mx_scales: list
        dn_nibbles: list
        dn_mx_scales: list

    out2, h2 = oracle.moe(MxLayer(E, H, I, gun, gus, dnn, dns), xb, ids, w, 32)
    assert np.array_equal(h1, h2) and np.array_equal(out1, out2)
