"""Pins for the oracle's products and bf16 rounding (CPU only).

The product is y = sum_k w[n][k] x[k] with w the decoded weight times its UE8M0 scale. The pins:
exact rational arithmetic (fractions), the correctly rounded sum (math.fsum), one-hot inputs,
the doubled-E2M1 integer identity from the "Tied Trit-Planes" page (section 2.3), and torch's
own float32 -> bf16 rounding for the oracle's bf16 rounding.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from trellis_coded_fp4_b200 import synth


def _case(rows, cols, T, seed, seg_len=32):
    st = synth.stream(rows, cols, seed)
    sc = synth.scales(rows, cols, seed)
    xb = synth.bf16_bits(synth.activations(T, cols, seed))
    return st, sc, xb


def test_gemv_equals_exact_rational_sum():
    rows, cols, T = 4, 96, 2
    for seg_len in (32, 96):
        st, sc, xb = _case(rows, cols, T, seed=21)
        y, wn = oracle.gemv(st, sc, rows, cols, seg_len, xb)
        w = oracle.decode_values(st, sc, rows, cols, seg_len)
        x = oracle.bf16_bits_to_f64(xb)
        for t in range(T):
            for n in range(rows):
                exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(w[n], x[t]))
                bound = cols * 2.0 ** -53 * float(np.abs(w[n] * x[t]).sum())
                assert abs(Fraction(y[t, n]) - exact) <= Fraction(bound)
                assert abs(y[t, n] - oracle.fsum_dot(w[n], x[t])) <= bound
        assert np.allclose(wn, np.sqrt((w * w).sum(axis=1)), rtol=0, atol=0)


def test_gemv_one_hot_returns_columns():
    rows, cols = 6, 64
    st, sc, _ = _case(rows, cols, 1, seed=22)
    w = oracle.decode_values(st, sc, rows, cols, 64)
    for k in (0, 1, 31, 32, 63):
        x = torch.zeros(1, cols, dtype=torch.bfloat16)
        x[0, k] = 1.0
        y, _ = oracle.gemv(st, sc, rows, cols, 64, synth.bf16_bits(x))
        assert (y[0] == w[:, k]).all()


def test_doubled_e2m1_integer_identity():
    # With every scale 127 (factor 1) and integer activations, 2*y is an exact integer sum of
    # doubled E2M1 magnitudes (integers 0..12) times signs times x.
    rows, cols = 5, 128
    st = synth.stream(rows, cols, seed=23)
    sc = np.full((rows, cols // 32), 127, np.uint8)
    xi = np.random.default_rng(23).integers(-8, 9, (1, cols))
    xb = synth.bf16_bits(torch.tensor(xi, dtype=torch.bfloat16))
    y, _ = oracle.gemv(st, sc, rows, cols, 32, xb)
    codes = oracle.decode_codes(st, rows, cols, 32)
    doubled = [0, 1, 2, 3, 4, 6, 8, 12]
    for n in range(rows):
        acc = 0
        for k in range(cols):
            c = int(codes[n, k])
            m = doubled[c & 7]
            acc += (-m if c & 8 else m) * int(xi[0, k])
        assert 2 * y[0, n] == acc


def test_gemv_row_subset_matches_full():
    rows, cols = 9, 64
    st, sc, xb = _case(rows, cols, 3, seed=24)
    y, wn = oracle.gemv(st, sc, rows, cols, 32, xb)
    ids = np.array([8, 0, 3])
    ys, wns = oracle.gemv(st, sc, rows, cols, 32, xb, row_ids=ids)
    assert (ys == y[:, ids]).all() and (wns == wn[ids]).all()


def test_bf16_round_matches_torch_float32_rounding():
    r = np.random.default_rng(25)
    vals = np.concatenate([
        r.standard_normal(20000).astype(np.float32),
        (r.standard_normal(2000) * 1e-39).astype(np.float32),       # bf16 subnormal range
        (r.standard_normal(2000) * 1e37).astype(np.float32),
    ])
    # exact ties: bf16 value plus half an ulp
    base = torch.from_numpy(r.standard_normal(2000).astype(np.float32)).to(torch.bfloat16)
    b32 = base.float().numpy().view(np.uint32)
    ties = (b32 | 0x8000).view(np.float32)
    vals = np.concatenate([vals, ties])
    ref = synth.bf16_bits(torch.from_numpy(vals).to(torch.bfloat16))
    ours = oracle.bf16_round_array(vals.astype(np.float64))
    assert (ours == ref).all()
    assert oracle.bf16_round(1e40) == float("inf")
