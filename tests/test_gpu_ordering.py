"""A product kernel launched right after a kernel that writes its weights reads the finished weights.

The GEMV's product kernels read their weights (stream words, scales, scale tiles, MXFP4 nibbles)
before their grid-dependency wait, and the activation split releases them early, so they may start
while earlier kernels still run. The library's kernels that write weights therefore release no
dependents early. Each case below writes a matrix over a buffer that held a different one and runs
the product on it in the same stream with no synchronisation in between; the outputs must be the
oracle's products of the newly written matrix (sampled rows, full tolerance and design bound).
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import synth

from gpu_common import assert_products_close, xnorms

pytestmark = pytest.mark.gpu

ROWS, COLS = 32 * 5760, 2880  # the stacked gate_up matrices of the 32-expert hidden-2880 layer


def _sample(rows, seed):
    return np.concatenate([[0, rows - 1], np.random.default_rng(seed).choice(rows, 126, replace=False)])


def test_gemv_right_after_repack_into_its_stream():
    g = torch.Generator(device="cuda")
    g.manual_seed(21)
    il = torch.randint(-2**31, 2**31 - 1, (ROWS, COLS // 32, 2), dtype=torch.int32, device="cuda", generator=g)
    planar = torch.randint(-2**31, 2**31 - 1, (ROWS, COLS // 32, 2), dtype=torch.int32, device="cuda", generator=g)
    sc = synth.scales(ROWS, COLS, 21)
    W = tc.TrellisMatrix(planar.reshape(-1), torch.from_numpy(sc.reshape(-1)).cuda(), ROWS, COLS, 32)
    x = synth.activations(1, COLS, seed=22)
    torch.cuda.synchronize()
    tc.repack_interleaved(il, ROWS, COLS, out=planar)  # overwrites W's stream
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    rows = _sample(ROWS, 23)
    idx = torch.from_numpy(rows).cuda()
    src = il[idx].cpu().numpy().view(np.uint32).reshape(len(rows), COLS // 32, 2)
    st = oracle.repack_interleaved(src, len(rows), COLS)
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(st, sc[rows], len(rows), COLS, 32, xb)
    assert_products_close(y[:, idx], y_exact, wn, xnorms(xb), "gemv after repack", cols=COLS)


def test_tiled_gemv_right_after_its_scale_tiles():
    layer = synth.moe_layer(32, 2880, 2880, seed=synth.SEED_BASE + 1)
    W = tc.TrellisMatrix.from_numpy(layer.gu_stream, layer.gu_scales, ROWS, COLS, 32)
    tiles = torch.full((tc.scale_tiles_bytes(W),), 0xFF, dtype=torch.uint8, device="cuda")  # NaN scales
    x = synth.activations(1, COLS, seed=24)
    torch.cuda.synchronize()
    tc.scale_tiles(W, out=tiles)
    y = tc.gemv_tiled(W, tiles, x.cuda())
    torch.cuda.synchronize()
    rows = _sample(ROWS, 25)
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(layer.gu_stream, layer.gu_scales, ROWS, COLS, 32, xb, row_ids=rows)
    assert_products_close(y[:, torch.from_numpy(rows).cuda()], y_exact, wn, xnorms(xb), "tiled gemv after tiles",
                          cols=COLS)


def test_mxfp4_gemv_right_after_the_expansion():
    layer = synth.moe_layer(32, 2880, 2880, seed=synth.SEED_BASE + 1)
    W = tc.TrellisMatrix.from_numpy(layer.gu_stream, layer.gu_scales, ROWS, COLS, 32)
    nib = torch.zeros((ROWS, COLS // 2), dtype=torch.uint8, device="cuda")
    osc = torch.full((ROWS, COLS // 32), 0xFF, dtype=torch.uint8, device="cuda")
    M = tc.Mxfp4Matrix(nib, osc, ROWS, COLS)
    x = synth.activations(1, COLS, seed=26)
    torch.cuda.synchronize()
    tc.decode_to_mxfp4(W, nib, osc)
    y = tc.mxfp4_gemv(M, x.cuda())
    torch.cuda.synchronize()
    rows = _sample(ROWS, 27)
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(layer.gu_stream, layer.gu_scales, ROWS, COLS, 32, xb, row_ids=rows)
    assert_products_close(y[:, torch.from_numpy(rows).cuda()], y_exact, wn, xnorms(xb), "mxfp4 gemv after expansion",
                          cols=COLS)


def test_gemv_right_after_the_encoder():
    rows, cols, seg = 4, 256, 32
    r = np.random.default_rng(28)
    sc = r.integers(120, 128, size=(rows, cols // 32), dtype=np.uint8)
    scale = np.repeat(2.0 ** (sc.astype(np.float64) - 127), 32, axis=1)
    target = r.normal(0, 2.5, (rows, cols)) * scale
    D = r.uniform(0.1, 10.0, (rows, cols))
    x = synth.activations(2, cols, seed=29)
    W0 = tc.TrellisMatrix.from_numpy(synth.stream(rows, cols, 30), sc, rows, cols, seg)
    torch.cuda.synchronize()
    W, _ = tc.encode(torch.from_numpy(target).cuda(), torch.from_numpy(D).cuda(), W0.scales, seg)
    y = tc.gemv(W, x.cuda())
    torch.cuda.synchronize()
    sym = np.zeros((rows, cols), np.uint8)
    for n in range(rows):
        for j in range(cols // seg):
            sl = slice(j * seg, (j + 1) * seg)
            sym[n, sl], _ = oracle.viterbi_encode(target[n, sl], D[n, sl], scale[n, sl])
    st = oracle.pack_symbols(sym, rows, cols)
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(st, sc, rows, cols, seg, xb)
    assert_products_close(y, y_exact, wn, xnorms(xb), "gemv after encode", cols=cols)
