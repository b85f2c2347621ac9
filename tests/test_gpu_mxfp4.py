"""GPU parity for the products read straight from a resident MXFP4 tensor (HEPH serving mode 2,
consumer side): mxfp4_gemv and mxfp4_grouped_moe against the oracle's MXFP4 products.

Inputs are seeded synthetic MXFP4 tensors (every E2M1 code, scales around 2^0) or the expansion of
synthetic trellis layers; expected values come from the oracle only. Tolerance as for the fused
paths: |y - exact| <= 2e-3 ||w_row|| ||x_t||.
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import _abi, synth

from gpu_common import (assert_products_close, bf16_to_f64, check_moe, half_ulp_bf16, mx_product, upload_matrix,
                        upload_mx, xnorms)

pytestmark = pytest.mark.gpu


def _random_mx(rows, cols, seed, lo=118, hi=130):
    rng = np.random.default_rng(seed)
    return (rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8),
            rng.integers(lo, hi, size=(rows, cols // 32), dtype=np.uint8))


@pytest.mark.parametrize("rows,cols,T", [(128, 64, 1), (200, 192, 3), (384, 1088, 5), (130, 2048, 6),
                                         (257, 640, 16), (64, 128, 32), (1000, 3072, 2)])
def test_mxfp4_gemv_small(rows, cols, T):
    # several 128-row tiles with a ragged last one, stages of 1024 / 512 K with a partial last
    # stage, both MMA widths (T <= 5 and T >= 6) and a second pass (T = 32)
    nib, sc = _random_mx(rows, cols, 7000 + rows + T)
    W = upload_mx(nib, sc)
    x = synth.activations(T, cols, seed=7000 + T).cuda()
    y = tc.mxfp4_gemv(W, x)
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x.cpu())
    ye, wn = oracle.mxfp4_gemv(nib, sc, rows, cols, xb)
    assert_products_close(y, ye, wn, xnorms(xb), f"mxfp4_gemv {rows}x{cols} T={T}", cols=cols)


def test_mxfp4_gemv_one_hot_returns_exact_elements():
    rows, cols = 300, 1024
    nib, sc = _random_mx(rows, cols, 7100, lo=120, hi=134)
    W = upload_mx(nib, sc)
    for k in (0, 1, 63, 64, 511, 1023):
        xb = np.zeros((1, cols), np.uint16)
        xb[0, k] = 0x3F80
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        y = tc.mxfp4_gemv(W, x)
        ye, _ = oracle.mxfp4_gemv(nib, sc, rows, cols, xb)
        got = oracle.bf16_bits_to_f64(synth.bf16_bits(y.cpu()))
        assert np.array_equal(got, ye), f"one-hot column {k}"


def test_mxfp4_gemv_of_expanded_trellis_matrix():
    # the mode-2 pipeline: expand a trellis matrix once on the GPU, then multiply from the tensor
    rows, cols, T = 2048, 2048, 4
    st, sc = synth.stream(rows, cols, 7200), synth.scales(rows, cols, 7200)
    Wt = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
    Wm = tc.Mxfp4Matrix.expand(Wt)
    x = synth.activations(T, cols, seed=7200).cuda()
    y = tc.mxfp4_gemv(Wm, x)
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x.cpu())
    ye, wn = oracle.gemv(st, sc, rows, cols, 32, xb)
    assert_products_close(y, ye, wn, xnorms(xb), "expanded 2048x2048", cols=cols)


@pytest.mark.parametrize("T", [1, 8])
def test_mxfp4_gemv_gate_up_size_sampled(T):
    # 32 experts' gate_up rows of the hidden-2880 layer (184320 x 2880) in one matrix; sampled rows
    rows, cols = 32 * 5760, 2880
    nib, sc = _random_mx(rows, cols, 7300 + T)
    W = upload_mx(nib, sc)
    x = synth.activations(T, cols, seed=7300 + T).cuda()
    y = tc.mxfp4_gemv(W, x)
    torch.cuda.synchronize()
    rid = np.sort(np.random.default_rng(T).choice(rows, 400, replace=False))
    xb = synth.bf16_bits(x.cpu())
    ye, wn = oracle.mxfp4_gemv(nib, sc, rows, cols, xb, row_ids=rid)
    assert_products_close(y[:, torch.from_numpy(rid).cuda()], ye, wn, xnorms(xb), "gate_up size", cols=cols)


def test_mxfp4_gemv_argument_errors():
    L = _abi.load()
    nib, sc = _random_mx(64, 128, 7400)
    W = upload_mx(nib, sc)
    x = synth.activations(1, 128, seed=1).cuda()
    y = torch.empty((1, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(tc.mxfp4_gemv_workspace_bytes(W, 1), dtype=torch.uint8, device="cuda")
    p = lambda t: t.data_ptr()
    bad_cols = _abi.Mxfp4(W.nibbles.data_ptr(), W.scales.data_ptr(), 64, 96)      # not a multiple of 64
    assert L.mxfp4_gemv(bad_cols, p(x), 1, p(y), p(ws), ws.numel(), None) == 3
    odd = _abi.Mxfp4(W.nibbles.data_ptr() + 8, W.scales.data_ptr(), 32, 128)     # nibbles not 16-aligned
    assert L.mxfp4_gemv(odd, p(x), 1, p(y), p(ws), ws.numel(), None) == 2
    odd_sc = _abi.Mxfp4(W.nibbles.data_ptr(), W.scales.data_ptr() + 1, 32, 128)  # odd scales
    assert L.mxfp4_gemv(odd_sc, p(x), 1, p(y), p(ws), ws.numel(), None) == 2
    assert L.mxfp4_gemv(W.abi(), p(x), 1, p(y), p(ws), ws.numel() - 1, None) == 4
    assert L.mxfp4_gemv(W.abi(), p(x), 33, p(y), p(ws), ws.numel(), None) == 3
    assert L.mxfp4_gemv(W.abi(), p(x), 0, p(y), None, 0, None) == 0
    torch.cuda.synchronize()


def _mx_layer(E, H, I, seed):
    return {"gu": [_random_mx(2 * I, H, seed + e) for e in range(E)],
            "dn": [_random_mx(H, I, seed + 1000 + e) for e in range(E)]}


def _mx_weights(mx, H, I):
    return tc.Mxfp4MoEWeights([upload_mx(*m) for m in mx["gu"]], [upload_mx(*m) for m in mx["dn"]], H, I)


class _Shape:
    def __init__(self, E, H, I):
        self.E, self.H, self.I = E, H, I


@pytest.mark.parametrize("T", [1, 3, 8])
def test_mxfp4_moe_small(T):
    E, H, I, k = 8, 128, 192, 2
    mx = _mx_layer(E, H, I, 7500 + T)
    W = _mx_weights(mx, H, I)
    x = synth.activations(T, H, seed=7500 + T).cuda()
    ids, wts = tc.moe_route(synth.logits(T, E, seed=7500 + T).cuda(), k)
    out, ws = tc.mxfp4_grouped_moe(W, x, ids, wts)
    torch.cuda.synchronize()
    check_moe(_Shape(E, H, I), W, x, ids, wts, out, ws, k, 32, product=mx_product(mx))


def test_mxfp4_moe_all_tokens_on_the_same_experts():
    E, H, I, k, T = 6, 256, 128, 3, 11
    mx = _mx_layer(E, H, I, 7600)
    W = _mx_weights(mx, H, I)
    ids = torch.tensor([[4, 1, 2]] * T, dtype=torch.int32).cuda()
    wts = torch.rand(T, k, generator=torch.Generator().manual_seed(7600)).cuda()
    x = synth.activations(T, H, seed=7600).cuda()
    out, ws = tc.mxfp4_grouped_moe(W, x, ids, wts)
    torch.cuda.synchronize()
    check_moe(_Shape(E, H, I), W, x, ids, wts, out, ws, k, 32, product=mx_product(mx))


def test_mxfp4_moe_32_experts_hidden_2880_expanded_batch1():
    # the mode-2 pipeline on the 32-expert hidden-2880 top-4 layer: expand every expert on the GPU
    # once, then the grouped MoE from the tensors; checked against the trellis layer's oracle
    E, H, I, k, T = 32, 2880, 2880, 4, 1
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 2)
    Wm = tc.Mxfp4MoEWeights.expand(tc.MoEWeights.from_layer(layer))
    x = synth.activations(T, H, seed=synth.SEED_BASE + 2).cuda()
    ids, wts = tc.moe_route(synth.logits(T, E, seed=synth.SEED_BASE + 2).cuda(), k)
    out, ws = tc.mxfp4_grouped_moe(Wm, x, ids, wts)
    torch.cuda.synchronize()
    check_moe(layer, Wm, x, ids, wts, out, ws, k, 32)


@pytest.mark.parametrize("T", [8, 32])
def test_mxfp4_moe_32_experts_batch_sweep_sampled(T):
    E, H, I, k = 32, 2880, 2880, 4
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 3)
    Wm = tc.Mxfp4MoEWeights.expand(tc.MoEWeights.from_layer(layer))
    x = synth.activations(T, H, seed=synth.SEED_BASE + 3 + T).cuda()
    ids, wts = tc.moe_route(synth.logits(T, E, seed=synth.SEED_BASE + 3 + T).cuda(), k)
    out, ws = tc.mxfp4_grouped_moe(Wm, x, ids, wts)
    torch.cuda.synchronize()
    r = np.random.default_rng(T)
    check_moe(layer, Wm, x, ids, wts, out, ws, k, 32, rows_h=r.choice(I, 48, replace=False),
              rows_out=r.choice(H, 48, replace=False))


def test_mxfp4_no_bounded_wait_gave_up():
    assert tc.device_timeouts() == 0


def _wide_range_activations(T, cols, seed):
    """bf16 activations whose 32-blocks each span ~2^-24 .. 2^6 with full 8-bit significands: the
    case where the six-term E2M1 split of a block has the most to do."""
    r = np.random.default_rng(seed)
    mant = 1.0 + r.integers(0, 128, (T, cols)) / 128.0
    expo = r.integers(-24, 7, (T, cols))
    sign = np.where(r.random((T, cols)) < 0.5, -1.0, 1.0)
    return torch.from_numpy(sign * mant * 2.0 ** expo).to(torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("T", [1, 5, 16])
def test_activation_split_within_its_bound(T):
    # Identity weights (E2M1 1.0 at [n][n], zeros elsewhere, scale 2^0) make y[t][n] the kernel's
    # reconstruction of x[t][n] from its E2M1 terms. Each element must lie within 5^-6 of its
    # block's largest magnitude (the six-term bound) plus half a bf16 ulp of the output; a split
    # with fewer terms, or terms dropped from the sum, misses it by orders of magnitude here.
    n = 1024
    nib = np.zeros((n, n // 2), np.uint8)
    idx = np.arange(n)
    nib[idx, idx // 2] = np.where(idx % 2 == 0, 0x02, 0x20).astype(np.uint8)  # E2M1 code 2 = +1.0
    sc = np.full((n, n // 32), 127, np.uint8)
    W = upload_mx(nib, sc)
    x = _wide_range_activations(T, n, 7600 + T)
    y = bf16_to_f64(tc.mxfp4_gemv(W, x.cuda()))
    torch.cuda.synchronize()
    xv = x.double().numpy()
    blk_max = np.repeat(np.abs(xv).reshape(T, n // 32, 32).max(axis=2), 32, axis=1)
    bound = 5.0 ** -6 * blk_max + half_ulp_bf16(np.maximum(np.abs(y), np.abs(xv)))
    bad = np.abs(y - xv) > bound
    assert not bad.any(), f"{bad.sum()} elements outside the split bound, first {np.argwhere(bad)[0].tolist()}"


@pytest.mark.parametrize("seg", [32, 2880])
def test_fused_gemv_wide_range_activations(seg):
    # the trellis GEMV on the same kind of activations, held to the design bound
    rows, cols, T = 300, 2880, 3
    st, sc, Wt = upload_matrix(rows, cols, seed=7700 + seg, seg_len=seg)
    x = _wide_range_activations(T, cols, 7700)
    y = tc.gemv(Wt, x.cuda())
    torch.cuda.synchronize()
    xb = synth.bf16_bits(x)
    ye, wn = oracle.gemv(st, sc, rows, cols, seg, xb)
    assert_products_close(y, ye, wn, xnorms(xb), f"wide-range x seg={seg}", cols=cols)
