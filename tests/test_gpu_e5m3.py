"""GPU parity for the E5M3 block-scale GEMV (trellis_gemv_e5m3) against the oracle, on both of its
paths: the tensor cores (cols a multiple of 64: four block-scaled MMAs per K-step, one per power of
two of the scale) and the CUDA cores (other shapes).

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
from gpu_common import assert_products_close, bf16_to_f64, xnorms

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


@pytest.mark.parametrize("seg", [32, 2880])
@pytest.mark.parametrize("T", [5, 16, 32])
def test_e5m3_tensor_cores_return_every_decoded_column(T, seg):
    # one-hot activations: every output is one decoded weight, an E2M1 value times an E5M3 scale (at
    # most 6 significant bits, exact in bf16), summed from its four power-of-two parts
    rows, cols = 300, 2880
    st, sc, W = _case(rows, cols, 950 + T + seg, seg)
    assert tc.gemv_e5m3_workspace_bytes(W, T) > 0
    w = oracle.decode_values(st, sc, rows, cols, seg, scale_fmt="e5m3")
    ys = []
    for k0 in range(0, cols, T):
        x = torch.zeros(T, cols, dtype=torch.bfloat16, device="cuda")
        n = min(T, cols - k0)
        x[torch.arange(n, device="cuda"), torch.arange(k0, k0 + n, device="cuda")] = 1.0
        ys.append(tc.gemv_e5m3(W, x)[:n])
    got = bf16_to_f64(torch.cat(ys))
    assert (got == w.T).all(), f"{(got != w.T).sum()} decoded weights differ"
    assert tc.device_timeouts() == 0


def test_zero_mantissa_is_bit_identical_to_ue8m0_on_tensor_cores():
    rows, cols, T = 64, 2880, 4
    st = synth.stream(rows, cols, 912)
    e = np.random.default_rng(912).integers(8, 15, (rows, cols // 32)).astype(np.uint8)
    W5 = tc.TrellisMatrix.from_numpy(st, (e << 3).astype(np.uint8), rows, cols, 32)
    W8 = tc.TrellisMatrix.from_numpy(st, (e + 112).astype(np.uint8), rows, cols, 32)
    x = synth.activations(T, cols, 913).cuda()
    assert tc.gemv_e5m3_workspace_bytes(W5, T) > 0 and tc.gemv_workspace_bytes(W8, T) > 0
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
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    g = lambda xp, T, yp, wsp=p(ws), wsb=ws.numel(): L.trellis_gemv_e5m3(W.abi(), xp, T, yp, wsp, wsb, None)  # noqa: E731
    assert g(p(x, 2), 1, p(y)) == 2   # misaligned x
    assert g(p(x), 33, p(y)) == 3     # T > 32
    assert g(p(x), -1, p(y)) == 1
    assert g(None, 1, p(y)) == 1
    assert g(p(x), 0, p(y)) == 0
    assert L.trellis_gemv_e5m3_workspace(W.abi(), 1) > 0     # cols 64: the tensor-core path
    assert g(p(x), 1, p(y), None, 0) == 4                    # ... which needs its workspace
    assert g(p(x), 1, p(y), p(ws, 16), ws.numel() - 16) == 2  # 256-byte aligned
    torch.cuda.synchronize()
