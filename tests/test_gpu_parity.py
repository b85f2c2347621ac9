"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the same inputs.

Bit-exact for the MXFP4 expansion (nibbles and scales); the stated tolerance
|y - exact| <= 2e-3 ||w_row|| ||x|| for products; exact ids for routing.
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import synth

from gpu_common import (assert_mostly_correctly_rounded, assert_products_close, bf16_to_f64, upload_matrix,
                        xnorms)

pytestmark = pytest.mark.gpu

SMALL = [(1, 32), (3, 64), (17, 96), (37, 1024), (128, 2880), (9, 7168)]


def _segs(cols):
    out = {32, cols}
    if cols % 64 == 0:
        out.add(64)
    return sorted(out)


# ----------------------------------------------------------------------------- expansion (mode 2)

@pytest.mark.parametrize("rows,cols", SMALL + [(5, 288), (1, 96)])
def test_expand_bit_exact_small(rows, cols):
    for seg in _segs(cols):
        st, sc, W = upload_matrix(rows, cols, seed=1000 + rows + cols, seg_len=seg)
        nib, osc = tc.decode_to_mxfp4(W)
        torch.cuda.synchronize()
        ref_nib, ref_sc = oracle.expand_mxfp4(st, sc, rows, cols, seg)
        assert (nib.cpu().numpy() == ref_nib).all(), (rows, cols, seg)
        assert (osc.cpu().numpy() == ref_sc).all()


def test_expand_unaligned_scale_pointers():
    rows, cols = 7, 160
    st, sc, W = upload_matrix(rows, cols, seed=77)
    big = torch.zeros(rows * cols // 32 + 1, dtype=torch.uint8, device="cuda")
    W.scales = torch.from_numpy(np.concatenate([np.zeros(1, np.uint8), sc.ravel()])).cuda()[1:]  # odd address
    out_sc = big[1:]
    nib, _ = tc.decode_to_mxfp4(W, out_scales=out_sc)
    torch.cuda.synchronize()
    ref_nib, ref_sc = oracle.expand_mxfp4(st, sc, rows, cols, 32)
    assert (nib.cpu().numpy() == ref_nib).all()
    assert (out_sc.cpu().numpy().reshape(rows, -1) == ref_sc).all()


def test_expand_output_16_byte_aligned_only():
    # an output 16 bytes past a 32-byte boundary takes the 16-byte stores instead of the 32-byte ones
    rows, cols = 9, 2880
    st, sc, W = upload_matrix(rows, cols, seed=78)
    buf = torch.zeros(rows * cols // 2 + 32, dtype=torch.uint8, device="cuda")
    assert buf.data_ptr() % 32 == 0
    out = buf[16:16 + rows * cols // 2].view(rows, cols // 2)
    nib, osc = tc.decode_to_mxfp4(W, out_nibbles=out)
    torch.cuda.synchronize()
    ref_nib, ref_sc = oracle.expand_mxfp4(st, sc, rows, cols, 32)
    assert (nib.cpu().numpy() == ref_nib).all() and (osc.cpu().numpy() == ref_sc).all()
    assert (buf[:16].cpu().numpy() == 0).all() and (buf[16 + rows * cols // 2:].cpu().numpy() == 0).all()


def test_expand_full_moe_layer_sampled():
    # The 32-expert, hidden-2880 layer (gate_up 32x5760x2880, down 32x2880x2880) in the launch
    # configuration the bench times: one call per kind; sampled rows checked bit-exactly, scales
    # checked in full.
    E, H, I = 32, 2880, 2880
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 1)
    r = np.random.default_rng(5)
    for st, sc, rows, cols in ((layer.gu_stream, layer.gu_scales, E * 2 * I, H),
                               (layer.dn_stream, layer.dn_scales, E * H, I)):
        W = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
        nib, osc = tc.decode_to_mxfp4(W)
        torch.cuda.synchronize()
        assert (osc.cpu().numpy().ravel() == sc.ravel()).all()
        sample = np.concatenate([[0, rows - 1], r.choice(rows, 62, replace=False)])
        st2 = st.reshape(rows, cols // 32, 2)[sample]
        sc2 = sc.reshape(rows, cols // 32)[sample]
        ref_nib, _ = oracle.expand_mxfp4(st2, sc2, len(sample), cols, 32)
        assert (nib[torch.from_numpy(sample).cuda()].cpu().numpy() == ref_nib).all()


# ----------------------------------------------------------------------------- fused GEMV (mode 1)

@pytest.mark.parametrize("rows,cols", SMALL)
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8, 32])
def test_gemv_small(rows, cols, T):
    for seg in _segs(cols):
        st, sc, W = upload_matrix(rows, cols, seed=2000 + rows + cols + T, seg_len=seg)
        x = synth.activations(T, cols, seed=2000 + T)
        y = tc.gemv(W, x.cuda())
        torch.cuda.synchronize()
        xb = synth.bf16_bits(x)
        y_exact, wn = oracle.gemv(st, sc, rows, cols, seg, xb)
        assert_products_close(y, y_exact, wn, xnorms(xb), f"{rows}x{cols} T={T} seg={seg}", cols=cols)


@pytest.mark.parametrize("seg", [64, 96, 160, 288, 480, 2880])
@pytest.mark.parametrize("T", [1, 6])
def test_gemv_long_segments_on_tensor_cores(seg, T):
    # K = 2880 (90 blocks): segments of 2, 3, 5, 9, 15 and 90 blocks start inside a decode thread's
    # 8 blocks, at a thread's first block and across stages; 300 rows leave a ragged last tile
    rows, cols = 300, 2880
    st, sc, W = upload_matrix(rows, cols, seed=2500 + seg + T, seg_len=seg)
    assert tc.gemv_workspace_bytes(W, T) > 0  # the tensor-core path takes it
    x = synth.activations(T, cols, seed=2500 + T)
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(st, sc, rows, cols, seg, xb)
    assert_products_close(y, y_exact, wn, xnorms(xb), f"seg={seg} T={T}", cols=cols)
    assert_mostly_correctly_rounded(y, y_exact, f"seg={seg} T={T}")


@pytest.mark.parametrize("seg", [32, 2048])
def test_gemv_2048_square_batch1(seg):
    rows = cols = 2048
    st, sc, W = upload_matrix(rows, cols, seed=synth.SEED_BASE + 0, seg_len=seg)
    x = synth.activations(1, cols, seed=synth.SEED_BASE + 0)
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(st, sc, rows, cols, seg, xb)
    assert_products_close(y, y_exact, wn, xnorms(xb), "2048^2", cols=cols)
    assert_mostly_correctly_rounded(y, y_exact, "2048^2")


@pytest.mark.parametrize("T", [1, 32])
def test_gemv_full_moe_layer_sampled(T):
    # Every expert matrix of the 32-expert hidden-2880 layer stacked (gate_up 184320 x 2880, down
    # 92160 x 2880): the shapes and launch configuration the bench times at T = 1 (register-split
    # instance), and T = 32 (the largest batch, one pass of the 192-row B operand). 64 sampled rows
    # per matrix against the oracle, plus every output finite.
    E, H, I = 32, 2880, 2880
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 1)
    r = np.random.default_rng(6 + T)
    x = synth.activations(T, H, seed=60 + T)
    xb = synth.bf16_bits(x)
    for st, sc, rows, cols in ((layer.gu_stream, layer.gu_scales, E * 2 * I, H),
                               (layer.dn_stream, layer.dn_scales, E * H, I)):
        W = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
        assert tc.gemv_workspace_bytes(W, T) > 0
        y = tc.gemv(W, x.cuda())
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all()
        sample = np.concatenate([[0, rows - 1], r.choice(rows, 62, replace=False)])
        y_exact, wn = oracle.gemv(st, sc, rows, cols, 32, xb, row_ids=sample)
        ys = y[:, torch.from_numpy(sample).cuda()]
        assert_products_close(ys, y_exact, wn, xnorms(xb), f"{rows}x{cols} T={T}", cols=cols)
        assert_mostly_correctly_rounded(ys, y_exact, f"{rows}x{cols} T={T}")


@pytest.mark.parametrize("T", [1, 32])
def test_gemv_largest_cols(T):
    # cols = 16384, the largest trellis_gemv takes (512 blocks, 16 stages per row)
    rows, cols = 130, 16384
    st, sc, W = upload_matrix(rows, cols, seed=2600 + T)
    x = synth.activations(T, cols, seed=2600 + T)
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(st, sc, rows, cols, 32, xb)
    assert_products_close(y, y_exact, wn, xnorms(xb), f"cols={cols} T={T}", cols=cols)


def test_gemv_one_hot_returns_exact_columns():
    rows, cols = 67, 256
    st, sc, W = upload_matrix(rows, cols, seed=31, seg_len=128)
    w = oracle.decode_values(st, sc, rows, cols, 128)
    ks = [0, 5, 31, 32, 100, 255]
    x = torch.zeros(len(ks), cols, dtype=torch.bfloat16)
    for t, k in enumerate(ks):
        x[t, k] = 1.0
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    assert (bf16_to_f64(y) == w[:, ks].T).all()


def test_gemv_unit_scale_integer_sums_are_exact():
    rows, cols = 33, 640
    st = synth.stream(rows, cols, seed=32)
    sc = np.full((rows, cols // 32), 127, np.uint8)
    W = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
    x = torch.ones(1, cols, dtype=torch.bfloat16)
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    exact, _ = oracle.gemv(st, sc, rows, cols, 32, synth.bf16_bits(x))
    ref = np.array([oracle.bf16_round(v) for v in exact[0]])
    assert (bf16_to_f64(y)[0] == ref).all()      # multiples of 0.5: fp32 sums are exact


# ----------------------------------------------------------------------------- routing

@pytest.mark.parametrize("T,E,k", [(1, 32, 4), (8, 32, 4), (32, 32, 4), (1, 256, 8), (32, 256, 8), (5, 8, 1),
                                   (3, 16, 8)])
def test_route(T, E, k):
    lg = synth.logits(T, E, seed=3000 + T + E + k)
    ids, w = tc.moe_route(lg.cuda(), k)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.route(lg.numpy(), k)
    assert (ids.cpu().numpy() == ref_ids).all()
    assert np.allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-7)


def test_route_nan_and_infinite_logits():
    # NaN ranks below every number and weighs as -inf; -inf best -> zero weights; +inf winners share
    nan, inf = float("nan"), float("inf")
    rows = [[nan, -inf, 1.0, nan], [nan, nan, nan, nan], [inf, 0.0, inf, -1.0], [-inf, -inf, nan, -inf],
            [2.0, nan, 2.0, 0.0]]
    lg = torch.tensor(rows, dtype=torch.float32)
    r = np.random.default_rng(44)
    lg2 = synth.logits(32, 256, seed=44)
    lg2[torch.from_numpy(r.random((32, 256)) < 0.5)] = nan
    for logits, k in ((lg, 3), (lg2, 8)):
        ids, w = tc.moe_route(logits.cuda(), k)
        torch.cuda.synchronize()
        ref_ids, ref_w = oracle.route(logits.numpy(), k)
        assert (ids.cpu().numpy() == ref_ids).all()
        assert np.allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-7)


def test_route_ties_go_to_lower_index():
    lg = torch.zeros(2, 16)
    lg[0, 3] = lg[0, 7] = lg[0, 11] = 2.0
    lg[1] = -1.0                                   # all equal
    ids, w = tc.moe_route(lg.cuda(), 4)
    torch.cuda.synchronize()
    assert ids.cpu().tolist() == [[3, 7, 11, 0], [0, 1, 2, 3]]
    assert np.allclose(w.cpu().numpy()[1], 0.25)
