"""GPU parity for the scale-tile path: trellis_make_scale_tiles (a permutation of the UE8M0 bytes,
checked against its layout restated in numpy) and trellis_gemv_tiled (against the oracle, bit for
bit against trellis_gemv, and as an exact column reader under one-hot activations)."""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import _abi, synth

from gpu_common import assert_mostly_correctly_rounded, assert_products_close, bf16_to_f64, upload_matrix, xnorms

pytestmark = pytest.mark.gpu


def _tiles_numpy(sc, rows, cols):
    """The scale-tile layout: tile t, group g, byte 16 r + 4 q + i = scale of row 128 t + 32 q + r,
    block 4 g + i (zero past the matrix); 8 groups per started 32 blocks."""
    nbr = cols // 32
    groups = 8 * ((nbr + 31) // 32)
    ntiles = (rows + 127) // 128
    pad = np.zeros((ntiles * 128, groups * 4), np.uint8)
    pad[:rows, :nbr] = sc.reshape(rows, nbr)
    # [t][q][r][g][i] -> [t][g][r][q][i]
    return pad.reshape(ntiles, 4, 32, groups, 4).transpose(0, 3, 2, 1, 4).reshape(-1)


@pytest.mark.parametrize("rows,cols", [(1, 64), (128, 1024), (300, 2880), (129, 1088), (77, 7168)])
def test_scale_tiles_layout(rows, cols):
    st, sc, W = upload_matrix(rows, cols, seed=8000 + rows)
    tiles = tc.scale_tiles(W)
    torch.cuda.synchronize()
    assert (tiles.cpu().numpy() == _tiles_numpy(sc, rows, cols)).all()


@pytest.mark.parametrize("rows,cols", [(37, 1024), (128, 2880), (300, 2880), (9, 7168), (130, 16384)])
@pytest.mark.parametrize("T", [1, 5, 6, 16, 32])
def test_gemv_tiled_matches_oracle_and_gemv(rows, cols, T):
    for seg in sorted({32, cols}):
        st, sc, W = upload_matrix(rows, cols, seed=8100 + rows + T, seg_len=seg)
        tiles = tc.scale_tiles(W)
        x = synth.activations(T, cols, seed=8100 + T)
        y = tc.gemv_tiled(W, tiles, x.cuda())
        y_ref = tc.gemv(W, x.cuda())
        torch.cuda.synchronize()
        xb = synth.bf16_bits(x)
        y_exact, wn = oracle.gemv(st, sc, rows, cols, seg, xb)
        assert_products_close(y, y_exact, wn, xnorms(xb), f"tiled {rows}x{cols} T={T} seg={seg}", cols=cols)
        assert (bf16_to_f64(y) == bf16_to_f64(y_ref)).all()  # the same products as the raw-scale path
    assert tc.device_timeouts() == 0


def test_gemv_tiled_full_size_sampled():
    # the stacked gate_up matrices of the 32-expert hidden-2880 layer, as the bench times it
    E, H, I = 32, 2880, 2880
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 1)
    rows = E * 2 * I
    W = tc.TrellisMatrix.from_numpy(layer.gu_stream, layer.gu_scales, rows, H, 32)
    tiles = tc.scale_tiles(W)
    x = synth.activations(1, H, seed=61)
    y = tc.gemv_tiled(W, tiles, x.cuda())
    torch.cuda.synchronize()
    sample = np.concatenate([[0, rows - 1], np.random.default_rng(9).choice(rows, 254, replace=False)])
    xb = synth.bf16_bits(x)
    y_exact, wn = oracle.gemv(layer.gu_stream, layer.gu_scales, rows, H, 32, xb, row_ids=sample)
    ys = y[:, torch.from_numpy(sample).cuda()]
    assert_products_close(ys, y_exact, wn, xnorms(xb), "tiled gate_up", cols=H)
    assert_mostly_correctly_rounded(ys, y_exact, "tiled gate_up")


@pytest.mark.parametrize("seg", [32, 2880])
@pytest.mark.parametrize("T", [5, 8, 16, 32])
def test_gemv_tiled_returns_every_decoded_column(T, seg):
    rows, cols = 300, 2880
    st, sc, W = upload_matrix(rows, cols, seed=8200 + T + seg, seg_len=seg)
    tiles = tc.scale_tiles(W)
    w = oracle.decode_values(st, sc, rows, cols, seg)
    ys = []
    for k0 in range(0, cols, T):
        x = torch.zeros(T, cols, dtype=torch.bfloat16, device="cuda")
        n = min(T, cols - k0)
        x[torch.arange(n, device="cuda"), torch.arange(k0, k0 + n, device="cuda")] = 1.0
        ys.append(tc.gemv_tiled(W, tiles, x)[:n])
    got = bf16_to_f64(torch.cat(ys))
    assert (got == w.T).all(), f"{(got != w.T).sum()} decoded weights differ"


def test_gemv_tiled_argument_errors():
    L = _abi.load()
    st, sc, W = upload_matrix(4, 96, seed=8300)   # 3 blocks per row: no tensor-core path
    tiles = tc.scale_tiles(W)
    x = torch.zeros((1, 96), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((1, 4), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    import ctypes
    vp = ctypes.c_void_p
    assert L.trellis_gemv_tiled(W.abi(), vp(tiles.data_ptr()), vp(x.data_ptr()), 1, vp(y.data_ptr()),
                                vp(ws.data_ptr()), ws.numel(), vp(s)) == 3   # cols not a multiple of 64
    st, sc, W = upload_matrix(4, 128, seed=8301)
    tiles = tc.scale_tiles(W)
    x = torch.zeros((1, 128), dtype=torch.bfloat16, device="cuda")
    assert L.trellis_gemv_tiled(W.abi(), vp(tiles.data_ptr()), vp(x.data_ptr()), 1, vp(y.data_ptr()),
                                vp(ws.data_ptr()), 16, vp(s)) == 4           # workspace too small
