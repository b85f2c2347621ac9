"""Pins for the oracle's D-weighted Viterbi encoder (CPU only).

"Curvature-aware Viterbi objective" bullet of the XOR-Trellis page: the search minimises
sum_k D_k (w_k - w_hat_k)^2 along trellis paths. Pins: the exhaustive minimum over all 4^L
sequences for L <= 8, exact round trips of decoded streams (the decoder is injective per
segment), and the scale invariance of the argmin in D.
"""
import numpy as np

import oracle
from trellis_coded_fp4_b200 import synth


def _cost(sym, target, D, scale):
    s, c = 0, 0.0
    for k, b in enumerate(sym):
        s = oracle.state_push(s, int(b))
        d = target[k] - oracle.state_value(s) * scale[k]
        c += D[k] * d * d
    return c


def test_viterbi_equals_bruteforce_minimum():
    r = np.random.default_rng(31)
    for L in range(1, 9):
        for _ in range(3):
            scale = 2.0 ** r.integers(-3, 2, L).astype(np.float64)
            target = r.normal(0, 3, L) * scale
            D = r.uniform(0.1, 10.0, L)
            sv, cv = oracle.viterbi_encode(target, D, scale)
            sb, cb = oracle.bruteforce_encode(target, D, scale)
            assert abs(cv - cb) <= 1e-12 * max(1.0, cb)
            assert abs(_cost(sv, target, D, scale) - cv) <= 1e-12 * max(1.0, cv)
            assert abs(_cost(sb, target, D, scale) - cb) <= 1e-12 * max(1.0, cb)


def test_encode_of_decoded_segment_round_trips():
    r = np.random.default_rng(32)
    for L in (32, 96):
        st = synth.stream(1, L, seed=32 + L)
        sc = synth.scales(1, L, seed=32 + L)
        w = oracle.decode_values(st, sc, 1, L, L)[0]
        scale = np.repeat(2.0 ** (sc[0].astype(np.float64) - 127), 32)
        D = r.uniform(0.01, 5.0, L)
        sym, cost = oracle.viterbi_encode(w, D, scale)
        assert cost == 0.0
        assert (oracle.pack_symbols(sym, 1, L) == st).all()


def test_argmin_invariant_to_scaling_D():
    r = np.random.default_rng(33)
    L = 24
    scale = np.full(L, 0.25)
    target = r.normal(0, 1.0, L)
    D = r.uniform(0.5, 2.0, L)
    s1, c1 = oracle.viterbi_encode(target, D, scale)
    s2, c2 = oracle.viterbi_encode(target, 8.0 * D, scale)
    assert (s1 == s2).all() and abs(c2 - 8.0 * c1) <= 1e-12 * c2


def test_large_D_weight_buys_accuracy_where_it_sits():
    # Raising D_k can only lower (or keep) the error at position k of the optimum.
    r = np.random.default_rng(34)
    L = 16
    scale = np.ones(L)
    target = r.normal(0, 2.0, L)
    D = np.ones(L)
    s1, _ = oracle.viterbi_encode(target, D, scale)
    D2 = D.copy()
    D2[7] = 1e6
    s2, _ = oracle.viterbi_encode(target, D2, scale)

    def err_at(sym, k):
        s = 0
        for i, b in enumerate(sym):
            s = oracle.state_push(s, int(b))
            if i == k:
                return abs(target[k] - oracle.state_value(s))

    assert err_at(s2, 7) <= err_at(s1, 7)
