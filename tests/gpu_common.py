"""Shared helpers for the GPU parity tests: upload synthetic inputs, compare with the oracle.

Tolerance for products (fp32 accumulation, bf16 out): |y_gpu - y_exact| <= 2e-3 ||w_row|| ||x_t||
per output, against the unrounded exact product (the stated target). A second, tighter check
holds the kernels to the error their own design allows:

    |y_gpu - y_exact| <= (sqrt(32) 5^-6 + 1.5 max((K/32 + 16) 2^-20, K 2^-24)) ||w|| ||x|| + ulp(y)/2

* sqrt(32) 5^-6: the tensor-core path writes each bf16 32-block of x as six E2M1 terms; every
  element is then off by at most 5^-6 of its block's largest magnitude, so the block's error
  vector has norm <= sqrt(32) 5^-6 ||x_block||;
* the fp32 accumulation, with room to spare: at most K/32 + 16 roundings of at most 2^-20 of the
  running sum on the tensor cores (blocks are summed exactly inside an MMA), or K roundings of
  2^-24 for the CUDA-core kernels' sequential FMA chain; the running sums are bounded by
  sum |w_k| sum_j |term_jk| <= 1.5 ||w|| ||x||;
* half a bf16 unit in the last place of the output.
"""
import numpy as np
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import synth

TOL = 2e-3


def tight_tol(cols):
    """The design's own relative bound for K = cols (the ulp term is added per output)."""
    return 32 ** 0.5 * 5.0 ** -6 + 1.5 * max((cols / 32 + 16) * 2.0 ** -20, cols * 2.0 ** -24)


def half_ulp_bf16(v):
    """Half a bf16 ulp at |v| (0 at v = 0)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def upload_matrix(rows, cols, seed, seg_len=32, lo=120, hi=126):
    st = synth.stream(rows, cols, seed)
    sc = synth.scales(rows, cols, seed, lo, hi)
    return st, sc, tc.TrellisMatrix.from_numpy(st, sc, rows, cols, seg_len)


def bf16_to_f64(t):
    return oracle.bf16_bits_to_f64(synth.bf16_bits(t.cpu()))


def assert_products_close(y_gpu, y_exact, wnorm, xnorm, what="", cols=None):
    """y_gpu: bf16 tensor [T][n]; y_exact [T][n] fp64; wnorm [n]; xnorm [T].
    cols: the reduction length K; when given, the design bound (module docstring) is checked too."""
    got = bf16_to_f64(y_gpu)
    wx = np.outer(xnorm, wnorm)
    bound = TOL * wx
    err = np.abs(got - y_exact)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} outputs out of tolerance; first {tuple(i)}: gpu {got[tuple(i)]!r} "
                             f"exact {y_exact[tuple(i)]!r} bound {bound[tuple(i)]!r}")
    if cols is not None:
        tight = tight_tol(cols) * wx + half_ulp_bf16(np.maximum(np.abs(got), np.abs(y_exact)))
        bad = err > tight
        if bad.any():
            i = np.argwhere(bad)[0]
            raise AssertionError(f"{what}: {bad.sum()} outputs outside the design bound; first {tuple(i)}: gpu "
                                 f"{got[tuple(i)]!r} exact {y_exact[tuple(i)]!r} bound {tight[tuple(i)]!r}")


def assert_mostly_correctly_rounded(y_gpu, y_exact, what="", max_frac=0.02):
    """For N(0,1) inputs the kernels' error is ~1e-6 of ||w|| ||x||, far below a bf16 ulp of y, so
    almost every output must be the correctly rounded exact product; an error the size of a
    dropped activation term or a wrong code in a small-scale block moves many of them."""
    got = bf16_to_f64(y_gpu)
    ref = torch.from_numpy(np.ascontiguousarray(y_exact)).to(torch.float32).to(torch.bfloat16).double().numpy()
    # y_exact -> fp32 is one extra rounding; only outputs within 2^-24 relative of a tie can differ
    frac = float((got != ref).mean())
    assert frac <= max_frac, f"{what}: {frac:.4f} of outputs are not the correctly rounded product"


def xnorms(x_bits):
    return np.linalg.norm(oracle.bf16_bits_to_f64(x_bits), axis=1)


def upload_mx(nib, sc):
    """A resident MXFP4 matrix from numpy nibbles [rows][cols/2] and scales [rows][cols/32]."""
    rows, half = nib.shape
    return tc.Mxfp4Matrix(torch.from_numpy(np.ascontiguousarray(nib)).cuda(),
                          torch.from_numpy(np.ascontiguousarray(sc)).cuda(), rows, 2 * half)


def _trellis_product(layer, kind, e, rows, cols, seg, xb, row_ids):
    return oracle.gemv(getattr(layer, kind + "_stream")[e], getattr(layer, kind + "_scales")[e], rows, cols, seg, xb,
                       row_ids=row_ids)


def mx_product(mx):
    """Oracle products of expert matrices given as MXFP4 numpy pairs: mx["gu"][e], mx["dn"][e]."""
    def product(layer, kind, e, rows, cols, seg, xb, row_ids):
        nib, sc = mx[kind][e]
        return oracle.mxfp4_gemv(nib, sc, rows, cols, xb, row_ids=row_ids)
    return product


def check_moe(layer, W, x, ids, wts, out, ws, k, seg_gu, seg_dn=None, rows_h=None, rows_out=None,
              product=_trellis_product):
    """Two-stage check of a grouped-MoE call.

    (i) h (read back from the workspace) against h_exact = silu(g) u from exact g, u, within the
        bound propagated from the product tolerance on g and u plus one bf16 rounding;
    (ii) out against sum_j w_j (down_j . h_gpu_j) computed exactly from the GPU's own h, within
        2e-3 sum_j |w_j| ||down_row|| ||h_j||.
    rows_h / rows_out: optional subsets of intermediate / output rows (sampled checks).
    product: the oracle's expert products (default: the trellis stream of `layer`)."""
    T = x.shape[0]
    H, I = layer.H, layer.I
    seg_dn = seg_gu if seg_dn is None else seg_dn
    x_bits = synth.bf16_bits(x.cpu())
    ids_np = ids.cpu().numpy()
    w_np = wts.cpu().numpy().astype(np.float64)
    off = W.hidden_offset(T, k)
    h_gpu = ws[off:off + T * k * I * 2].view(torch.int16).cpu().numpy().view(np.uint16).reshape(T, k, I)
    ri = np.arange(I) if rows_h is None else np.asarray(rows_h)
    rn = np.arange(H) if rows_out is None else np.asarray(rows_out)
    xn = xnorms(x_bits)
    for t in range(T):
        for j in range(k):
            e = int(ids_np[t, j])
            if not 0 <= e < layer.E:
                continue
            gu_rows = np.concatenate([ri, I + ri])
            y, wn = product(layer, "gu", e, 2 * I, H, seg_gu, x_bits[t:t + 1], gu_rows)
            g, u = y[0, :len(ri)], y[0, len(ri):]
            dg, du = TOL * wn[:len(ri)] * xn[t], TOL * wn[len(ri):] * xn[t]
            sg = oracle.silu(g)
            h_exact = sg * u
            bound = 1.1 * np.abs(u) * dg + (np.abs(sg) + 1.1 * dg) * du + 2.0 ** -8 * np.abs(h_exact) + 1e-30
            h_got = oracle.bf16_bits_to_f64(h_gpu[t, j, ri])
            bad = np.abs(h_got - h_exact) > bound
            assert not bad.any(), f"h out of bound at t={t} j={j} rows {ri[bad][:5]}"
    out_got = bf16_to_f64(out)
    for t in range(T):
        acc = np.zeros(len(rn))
        bnd = np.zeros(len(rn))
        for j in range(k):
            e = int(ids_np[t, j])
            if not 0 <= e < layer.E:
                continue
            hb = h_gpu[t, j][None, :]
            y, wn = product(layer, "dn", e, H, I, seg_dn, hb, rn)
            acc += w_np[t, j] * y[0]
            bnd += abs(w_np[t, j]) * wn * np.linalg.norm(oracle.bf16_bits_to_f64(hb))
        bad = np.abs(out_got[t, rn] - acc) > TOL * bnd + 1e-30
        assert not bad.any(), f"out out of bound at t={t} rows {rn[bad][:5]}"
