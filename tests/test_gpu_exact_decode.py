"""Bit-exact decode inside the fused product kernels, at full K, through every kernel instance.

A one-hot activation row e_k turns each product kernel into a column reader: the single non-zero
activation 1.0 is one E2M1 term with no residual, every product but one is an exact zero, and the
remaining one is a decoded weight, an E2M1 value times a power of two that bf16 holds exactly. So
y[t] must EQUAL column k_t of the decoded matrix, element for element. Sweeping k over every
column checks every decoded code and every scale of the matrix as the kernel uses them, with the
decode running in TMEM-feeding decode warps of the tensor-core kernel (the XOR-Trellis news page's
decoder bullet; HEPH's grid-aligned scales), not in a separate decoder.

Instances covered (each is its own template instance of the product kernel):
  * up to five tokens per call: the 32-row B operand with two MMA issuers and the register split;
  * 6-10 tokens: the 64-row B operand, 32-block stages, one issuer;
  * 11-16 tokens: the 96-row B operand, 16-block stages;
  * 17-32 tokens: the 192-row B operand with one accumulator;
  * each of the above for 32-weight segments and for one segment per row (state carried across
    blocks and stages);
  * the resident-MXFP4 source mode (products from the expanded tensor);
  * the grouped MoE: gate/up (through h = bf16(silu(g) u), which a wrong code moves by far more than
    its rounding) and down (through a one-hot h, which makes each output one exact product).
rows = 300 leaves a ragged last 128-row tile; cols = 2880 (90 blocks) a ragged last stage.
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import synth

from gpu_common import bf16_to_f64, upload_matrix

pytestmark = pytest.mark.gpu

ROWS, COLS = 300, 2880


def _one_hot_sweep(fn, cols, T, rows):
    """y for one-hot activations over every column, T columns per call: [cols][rows] fp64."""
    ys = []
    for k0 in range(0, cols, T):
        x = torch.zeros(T, cols, dtype=torch.bfloat16, device="cuda")
        n = min(T, cols - k0)
        x[torch.arange(n, device="cuda"), torch.arange(k0, k0 + n, device="cuda")] = 1.0
        ys.append(fn(x)[:n])
    y = torch.cat(ys)
    torch.cuda.synchronize()
    return bf16_to_f64(y)


def _assert_columns(got, w, what):
    ref = w.T  # [cols][rows]
    bad = got != ref
    if bad.any():
        k, n = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} decoded weights differ; first column {k} row {n}: "
                             f"kernel {got[k, n]!r}, decoded {ref[k, n]!r}")


@pytest.mark.parametrize("seg", [32, COLS])
@pytest.mark.parametrize("T", [5, 8, 16, 32])
def test_fused_gemv_returns_every_decoded_column(T, seg):
    st, sc, W = upload_matrix(ROWS, COLS, seed=5100 + T + seg, seg_len=seg)
    assert tc.gemv_workspace_bytes(W, T) > 0  # the tensor-core path
    w = oracle.decode_values(st, sc, ROWS, COLS, seg)
    got = _one_hot_sweep(lambda x: tc.gemv(W, x), COLS, T, ROWS)
    _assert_columns(got, w, f"trellis_gemv T={T} seg={seg}")
    assert tc.device_timeouts() == 0


@pytest.mark.parametrize("T", [1])
def test_fused_gemv_single_token_calls(T):
    # the batch-1 call itself (one token per launch), on a smaller column range to bound the calls
    rows, cols = 130, 640
    st, sc, W = upload_matrix(rows, cols, seed=5150)
    w = oracle.decode_values(st, sc, rows, cols, 32)
    got = _one_hot_sweep(lambda x: tc.gemv(W, x), cols, T, rows)
    _assert_columns(got, w, "trellis_gemv T=1")


@pytest.mark.parametrize("T", [5, 16])
def test_mxfp4_gemv_returns_every_decoded_column(T):
    st, sc, W = upload_matrix(ROWS, COLS, seed=5200 + T)
    nib, osc = oracle.expand_mxfp4(st, sc, ROWS, COLS, 32)
    M = tc.Mxfp4Matrix(torch.from_numpy(nib).cuda(), torch.from_numpy(osc).cuda(), ROWS, COLS)
    w = oracle.decode_values(st, sc, ROWS, COLS, 32)
    got = _one_hot_sweep(lambda x: tc.mxfp4_gemv(M, x), COLS, T, ROWS)
    _assert_columns(got, w, f"mxfp4_gemv T={T}")


# ----------------------------------------------------------------------------- grouped MoE

H = I = 2880


def _moe_layer(seg, mx, seed):
    layer = synth.moe_layer(2, H, I, seed=seed)
    W = tc.MoEWeights.from_layer(layer, seg_len=seg, seg_len_down=seg)
    run = tc.grouped_moe
    if mx:
        W = tc.Mxfp4MoEWeights.expand(W)
        run = tc.mxfp4_grouped_moe
    return layer, W, run


def _gu_scales(W, mx):
    return W.gate_up[1].scales


@pytest.mark.parametrize("mx", [False, True])
@pytest.mark.parametrize("seg", [32, "row"])
@pytest.mark.parametrize("T", [5, 16])
def test_moe_gate_up_decodes_every_column(T, seg, mx):
    # Every token on expert 1 (k = 1, weight 1), token t one-hot at column k_t: g and u are the
    # decoded weights gate[i][k_t] and up[i][k_t] exactly, so h must be bf16(silu(g) u) to within its
    # one rounding (the kernel's fp32 silu adds ~1e-7 relative). A wrong code changes g or u by at
    # least a quarter of its value, far outside that, unless the other factor is zero.
    if mx and seg != 32:
        pytest.skip("the MXFP4 layer has no trellis segments")
    s = H if seg == "row" else 32
    layer, W, run = _moe_layer(s, mx, seed=5300 + T)
    wg = oracle.decode_values(layer.gu_stream[1], layer.gu_scales[1], 2 * I, H, s)
    ids = torch.ones(T, 1, dtype=torch.int32, device="cuda")
    wts = torch.ones(T, 1, dtype=torch.float32, device="cuda")
    off = W.hidden_offset(T, 1)
    hs = []
    for k0 in range(0, H, T):
        x = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
        n = min(T, H - k0)
        x[torch.arange(n, device="cuda"), torch.arange(k0, k0 + n, device="cuda")] = 1.0
        _, ws = run(W, x, ids, wts)
        hs.append(ws[off:off + T * I * 2].view(torch.int16).view(T, I)[:n].clone())
    h = oracle.bf16_bits_to_f64(torch.cat(hs).cpu().numpy().view(np.uint16))  # [H][I]
    g, u = wg[:I].T, wg[I:].T                                                  # [H][I]
    exact = oracle.silu(g) * u
    bound = 2.0 ** -8 * np.abs(exact) * (1 + 2.0 ** -10) + 1e-40
    bad = np.abs(h - exact) > bound
    assert not bad.any(), f"h off at {np.argwhere(bad)[:3].tolist()} of {bad.sum()}"
    assert tc.device_timeouts() == 0


@pytest.mark.parametrize("mx", [False, True])
@pytest.mark.parametrize("seg", [32, "row"])
def test_moe_down_decodes_every_column(seg, mx):
    # One token on expert 1 (k = 1, weight 1). Zero UE8M0 bytes on every gate/up row but i and
    # I + i make every other h element round to zero (the products are ~2^-125, h ~2^-250), and a
    # one-hot x at a column where gate[i] and up[i] are non-zero makes h[i] non-zero: h is one-hot,
    # its split into E2M1 terms is exact, and out[n] = bf16(down[n][i] * h[i]) exactly (10
    # significant bits in fp32, one rounding). Sweeping i checks every decoded column of down.
    if mx and seg != 32:
        pytest.skip("the MXFP4 layer has no trellis segments")
    s = H if seg == "row" else 32
    layer, W, run = _moe_layer(s, mx, seed=5400)
    wg = oracle.decode_values(layer.gu_stream[1], layer.gu_scales[1], 2 * I, H, s)
    wd = oracle.decode_values(layer.dn_stream[1], layer.dn_scales[1], H, I, s)
    sc = _gu_scales(W, mx)
    orig = sc.clone().view(2 * I, H // 32)
    view = sc.view(2 * I, H // 32)
    ids = torch.ones(1, 1, dtype=torch.int32, device="cuda")
    wts = torch.ones(1, 1, dtype=torch.float32, device="cuda")
    off = W.hidden_offset(1, 1)
    both = (wg[:I] != 0) & (wg[I:] != 0)  # [I][H]: columns where gate and up are non-zero
    outs, hs = [], []
    view.zero_()
    for i in range(I):
        k = int(np.argmax(both[i]))
        assert both[i, k]
        view[i] = orig[i]
        view[I + i] = orig[I + i]
        x = torch.zeros(1, H, dtype=torch.bfloat16, device="cuda")
        x[0, k] = 1.0
        out, ws = run(W, x, ids, wts)
        outs.append(out.clone())
        hs.append(ws[off:off + I * 2].view(torch.int16).clone())
        view[i] = 0
        view[I + i] = 0
    view.copy_(orig)
    out = bf16_to_f64(torch.cat(outs))                                           # [I][H]
    h = oracle.bf16_bits_to_f64(torch.stack(hs).cpu().numpy().view(np.uint16))  # [I][I]
    hi = np.diag(h).copy()
    off_diag = h.copy()
    np.fill_diagonal(off_diag, 0)
    assert (off_diag == 0).all() and (hi != 0).all(), "h is not one-hot"
    # each product has at most 10 significant bits, so it is exact in fp32 and torch's
    # round-to-nearest-even conversion gives its bf16 rounding
    prod = torch.from_numpy(hi[:, None] * wd.T).to(torch.float32)
    assert (prod.double().numpy() == hi[:, None] * wd.T).all()
    ref = prod.to(torch.bfloat16).double().numpy()                                  # [I][H]
    bad = out != ref
    assert not bad.any(), f"down output differs at {np.argwhere(bad)[:3].tolist()} of {bad.sum()}"
    assert tc.device_timeouts() == 0
