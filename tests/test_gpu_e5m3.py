"""GPU parity for the E5M3 block-scale GEMV (trellis_gemv_e5m3, CUDA-core kernel) against the oracle.

The XOR-Trellis news page pairs E2M1 elements with E5M3 block scales; the encoding is the reading
in tests/golden/e5m3_reading.txt. Tolerance as for every product here:
|y_gpu - y_exact| <= 2e-3 ||w_row||_2 ||x_t||_2 against the unrounded exact product.
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import _abi, synth
from gpu_common import assert_products_close, xnorms

pytestmark = pytest.mark.gpu


def _case(rows, cols, seed, seg):
    st = synth.stream(rows, cols, seed)
    # exponents 8..14 (2^-7 .. 2^-1, the magnitudes of the UE8M0 workloads), any mantissa
    sc = np.random.default_rng(seed).integers(0x40, 0x78, (rows, cols // 32)).astype(np.uint8)
    return st, sc, tc.TrellisMatrix.from_numpy(st, sc, rows, cols, seg)


@pytest.mark.parametrize("rows,cols", [(37, 96), (130, 2880), (9, 4096)])
@pytest.mark.parametrize("T", [1, 3, 8, 32])
def test_e5m3_gemv_matches_oracle(rows, cols, T):
    for seg in (32, cols):
        st, sc, W = _case(rows, cols, 900 + rows + T, seg)
        x = synth.activations(T, cols, 901 + T).cuda()
        y = tc.gemv_e5m3(W, x)
        torch.cuda.synchronize()
        xb = synth.bf16_bits(x.cpu())
        y_ex, wn = oracle.gemv(st, sc, rows, cols, seg, xb, scale_fmt="e5m3")
        assert_products_close(y, y_ex, wn, xnorms(xb), f"e5m3 {rows}x{cols} T={T} seg={seg}", cols=cols)


def test_zero_mantissa_is_bit_identical_to_ue8m0():
    # cols = 96 (not a multiple of 64) keeps trellis_gemv on the same CUDA-core kernel; with zero
    # mantissas both calls scale by the same powers of two
    rows, cols, T = 50, 96, 4
    st = synth.stream(rows, cols, 910)
    e = np.random.default_rng(910).integers(1, 31, (rows, cols // 32)).astype(np.uint8)
    W5 = tc.TrellisMatrix.from_numpy(st, (e << 3).astype(np.uint8), rows, cols, 32)
    W8 = tc.TrellisMatrix.from_numpy(st, (e + 112).astype(np.uint8), rows, cols, 32)
    x = synth.activations(T, cols, 911).cuda()
    assert tc.gemv_workspace_bytes(W8, T) == 0
    y5, y8 = tc.gemv_e5m3(W5, x), tc.gemv(W8, x)
    torch.cuda.synchronize()
    assert torch.equal(y5.view(torch.int16), y8.view(torch.int16))


def test_nan_scale_propagates():
    rows, cols = 4, 64
    st, sc, _ = _case(rows, cols, 920, 32)
    sc[2, 1] = 0xF8
    W = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
    x = synth.activations(1, cols, 921).cuda()
    y = tc.gemv_e5m3(W, x).float().cpu().numpy()
    y_ex, _ = oracle.gemv(st, sc, rows, cols, 32, synth.bf16_bits(x.cpu()), scale_fmt="e5m3")
    assert np.isnan(y[0, 2]) and np.isnan(y_ex[0, 2])
    assert not np.isnan(y[0, [0, 1, 3]]).any()


def test_e5m3_full_size_sampled():
    # 184320 x 2880 (the gate/up matrices of the 32-expert hidden-2880 layer stacked) at batch 1, as
    # the bench times it; 64 sampled rows against the oracle
    rows, cols = 32 * 5760, 2880
    st = synth.stream(rows, cols, 930)
    sc = np.random.default_rng(930).integers(0x40, 0x78, (rows, cols // 32)).astype(np.uint8)
    W = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
    x = synth.activations(1, cols, 931).cuda()
    y = tc.gemv_e5m3(W, x)
    torch.cuda.synchronize()
    sample = np.concatenate([[0, rows - 1], np.random.default_rng(4).choice(rows, 62, replace=False)])
    xb = synth.bf16_bits(x.cpu())
    y_ex, wn = oracle.gemv(st, sc, rows, cols, 32, xb, row_ids=sample, scale_fmt="e5m3")
    assert_products_close(y[:, torch.from_numpy(sample).cuda()], y_ex, wn, xnorms(xb), "e5m3 full size",
                          cols=cols)


def test_e5m3_argument_errors():
    L = _abi.load()
    st, sc, W = _case(2, 64, 940, 32)
    x = torch.zeros((40, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((40, 2), dtype=torch.bfloat16, device="cuda")
    p = lambda t, off=0: t.data_ptr() + off
    assert L.trellis_gemv_e5m3(W.abi(), p(x, 2), 1, p(y), None) == 2   # misaligned x
    assert L.trellis_gemv_e5m3(W.abi(), p(x), 33, p(y), None) == 3     # T > 32
    assert L.trellis_gemv_e5m3(W.abi(), p(x), -1, p(y), None) == 1
    assert L.trellis_gemv_e5m3(W.abi(), None, 1, p(y), None) == 1
    assert L.trellis_gemv_e5m3(W.abi(), p(x), 0, p(y), None) == 0
    torch.cuda.synchronize()
