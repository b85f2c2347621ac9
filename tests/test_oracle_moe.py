"""Pins for the oracle's routing and MoE composition (CPU only).

Routing (top-k, softmax over the selected logits) is checked against numpy's stable argsort and
scipy's softmax. The layer is checked against a dense numpy MLP built from the decoded weights
(k = 1) and against the identity "identical experts give the single-expert output".
"""
import numpy as np
import scipy.special
import oracle
from trellis_coded_fp4_b200 import synth


def test_route_matches_stable_argsort_and_softmax():
    lg = synth.logits(16, 32, seed=41).numpy().astype(np.float64)
    lg[3, 5] = lg[3, 9] = 10.0                      # a tie: lower index first
    for k in (1, 4, 8):
        ids, w = oracle.route(lg, k)
        ref = np.argsort(-lg, axis=1, kind="stable")[:, :k]
        assert (ids == ref).all()
        sel = np.take_along_axis(lg, ref, axis=1)
        assert np.allclose(w, scipy.special.softmax(sel, axis=1), rtol=1e-15, atol=0)
    _, wall = oracle.route(lg, 32)
    assert np.allclose(np.sort(wall, axis=1), np.sort(scipy.special.softmax(lg, axis=1), axis=1))
    assert oracle.route(lg, 4)[0][3, 0] == 5 and oracle.route(lg, 4)[0][3, 1] == 9


def test_route_nan_and_infinite_logits():
    # hand-worked cases of the reading: NaN ranks below every number (-inf included) and weighs as
    # -inf; a token whose best selected logit is -inf gets zero weights; +inf winners share equally
    nan, inf = np.nan, np.inf
    lg = np.array([[nan, -inf, 1.0, nan],
                   [nan, nan, nan, nan],
                   [inf, 0.0, inf, -1.0],
                   [-inf, -inf, nan, -inf],
                   [2.0, nan, 2.0, 0.0]])
    ids, w = oracle.route(lg, 3)
    assert ids.tolist() == [[2, 1, 0], [0, 1, 2], [0, 2, 1], [0, 1, 3], [0, 2, 3]]
    assert w[0].tolist() == [1.0, 0.0, 0.0]
    assert w[1].tolist() == [0.0, 0.0, 0.0] and w[3].tolist() == [0.0, 0.0, 0.0]
    assert w[2].tolist() == [0.5, 0.5, 0.0]
    assert np.allclose(w[4], scipy.special.softmax([2.0, 2.0, 0.0]), rtol=1e-15, atol=0)
    # random NaN placement: ranking equals a lexicographic sort on (is NaN, -logit, index)
    lg = synth.logits(8, 32, seed=43).numpy().astype(np.float64)
    lg[np.random.default_rng(43).random(lg.shape) < 0.3] = nan
    for k in (1, 4, 8):
        ids, w = oracle.route(lg, k)
        for t in range(lg.shape[0]):
            ref = np.lexsort((np.arange(32), -np.nan_to_num(lg[t], nan=0.0), np.isnan(lg[t])))[:k]
            assert ids[t].tolist() == ref.tolist()
            sel = np.where(np.isnan(lg[t, ref]), -inf, lg[t, ref])
            assert np.allclose(w[t], scipy.special.softmax(sel), rtol=1e-15, atol=0)


def _dense_mlp(layer, e, x_bits, seg_len):
    """Decoded down matrix and the exact gate/up products of expert e, by numpy matmul."""
    H, I = layer.H, layer.I
    Wgu = oracle.decode_values(layer.gu_stream[e], layer.gu_scales[e], 2 * I, H, seg_len)
    Wdn = oracle.decode_values(layer.dn_stream[e], layer.dn_scales[e], H, I, seg_len)
    gu = Wgu @ oracle.bf16_bits_to_f64(x_bits)
    return Wdn, gu[:I], gu[I:]


def test_moe_single_expert_is_dense_mlp():
    E, H, I = 3, 64, 96
    layer = synth.moe_layer(E, H, I, seed=42)
    xb = synth.bf16_bits(synth.activations(2, H, seed=42))
    ids = np.array([[2], [0]], np.int32)
    w = np.ones((2, 1))
    out, h_bits = oracle.moe(layer, xb, ids, w, 32)
    for t in range(2):
        Wdn, g, u = _dense_mlp(layer, int(ids[t, 0]), xb[t], 32)
        h = oracle.bf16_bits_to_f64(h_bits[t, 0])
        ref_h = g / (1 + np.exp(-g)) * u
        ulp = np.abs(ref_h) * 2.0 ** -8 + 1e-300
        assert (np.abs(h - ref_h) <= ulp).all()      # h is ref_h rounded to bf16
        assert np.allclose(out[t], Wdn @ h, rtol=1e-12, atol=1e-12)


def test_moe_identical_experts_reduce_to_one():
    E, H, I, k = 4, 64, 64, 3
    layer = synth.moe_layer(E, H, I, seed=43)
    for arr in (layer.gu_stream, layer.gu_scales, layer.dn_stream, layer.dn_scales):
        arr[:] = arr[0]
    xb = synth.bf16_bits(synth.activations(3, H, seed=43))
    lg = synth.logits(3, E, seed=43).numpy()
    ids, w = oracle.route(lg, k)
    out, _ = oracle.moe(layer, xb, ids, w, 64)
    single, _ = oracle.moe(layer, xb, ids[:, :1], np.ones((3, 1)), 64)
    assert np.allclose(out, single, rtol=1e-12, atol=1e-12)


def test_silu_special_values():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(50.0) == 50.0
    assert abs(oracle.silu(-50.0)) < 1e-19
    assert np.isclose(oracle.silu(1.0), 1.0 / (1.0 + np.exp(-1.0)))
