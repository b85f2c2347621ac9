"""CPU oracle for trellis-coded FP4: decode, MXFP4 expansion, products, routing, MoE layer.

TEST INFRASTRUCTURE. Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA library and never calls it.

The per-weight work (decoder, expansion, products, Viterbi) is plain C in ``tcf4_oracle.c``;
this module loads it with ctypes and composes routing and the MoE layer in numpy fp64:

* routing — "top-k selection and softmax weights" as the routed-MoE workloads state it: the k
  largest logits (ties to the lower expert index), softmax over the selected k, in fp64;
* MoE layer — per selected expert j of token t: gate_up product, h = bf16(silu(g) * u) with
  g = rows 0..I-1 and u = rows I..2I-1, down product, out = sum_j w_j * y_j in fp64. The
  SwiGLU form (gate rows first, no clamp, no bias) is a reading; the pages name only a
  "fused grouped-MoE" ("HEPH" abstract) and a "SwiGLU epilogue" (fused-Hadamard news page).

Pins: every function here is checked by ``tests/test_oracle_*.py`` against something other than
itself (printed constants, E2M1 definitions, brute force, exact rational sums, closed forms).
The bit conventions of the stream (symbol bit order, palette/permutation bit order, planar
packing) are readings the pages do not fix: parity unpinned for those conventions alone.
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


def lib():
    """The loaded oracle library (built on first use)."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        u8p, u16p, u32p = P(ctypes.c_uint8), P(ctypes.c_uint16), P(ctypes.c_uint32)
        f64p, i64p, i64 = P(ctypes.c_double), P(ctypes.c_int64), ctypes.c_int64
        L.oracle_tables.argtypes = [f64p, u32p]
        L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_ue8m0_value.argtypes = [ctypes.c_uint8]
        L.oracle_ue8m0_value.restype = ctypes.c_double
        L.oracle_e5m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e5m3_value.restype = ctypes.c_double
        L.oracle_decode_values_e5m3.argtypes = [u32p, u8p, i64, i64, i64, f64p]
        L.oracle_gemv_e5m3.argtypes = [u32p, u8p, i64, i64, i64, u16p, i64, i64p, i64, f64p, f64p]
        L.oracle_state_push.argtypes = [ctypes.c_uint32, ctypes.c_uint32]
        L.oracle_state_push.restype = ctypes.c_uint32
        L.oracle_state_decode.argtypes = [ctypes.c_uint32, P(ctypes.c_int), P(ctypes.c_int)]
        L.oracle_state_value.argtypes = [ctypes.c_uint32]
        L.oracle_state_value.restype = ctypes.c_double
        L.oracle_state_code.argtypes = [ctypes.c_uint32]
        L.oracle_state_code.restype = ctypes.c_uint8
        L.oracle_decode_codes.argtypes = [u32p, i64, i64, i64, u8p]
        L.oracle_decode_values.argtypes = [u32p, u8p, i64, i64, i64, f64p]
        L.oracle_expand_mxfp4.argtypes = [u32p, u8p, i64, i64, i64, u8p, u8p]
        L.oracle_decode_codes_interleaved.argtypes = [u32p, i64, i64, i64, u8p]
        L.oracle_repack_interleaved.argtypes = [u32p, i64, i64, u32p]
        L.oracle_mxfp4_gemv.argtypes = [u8p, u8p, i64, i64, u16p, i64, i64p, i64, f64p, f64p]
        L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_value.restype = ctypes.c_double
        L.oracle_bf16_round.argtypes = [ctypes.c_double]
        L.oracle_bf16_round.restype = ctypes.c_double
        L.oracle_bf16_bits.argtypes = [ctypes.c_double]
        L.oracle_bf16_bits.restype = ctypes.c_uint16
        L.oracle_gemv.argtypes = [u32p, u8p, i64, i64, i64, u16p, i64, i64p, i64, f64p, f64p]
        L.oracle_viterbi_encode.argtypes = [f64p, f64p, f64p, i64, u8p]
        L.oracle_viterbi_encode.restype = ctypes.c_double
        L.oracle_bruteforce_encode.argtypes = [f64p, f64p, f64p, i64, u8p]
        L.oracle_bruteforce_encode.restype = ctypes.c_double
        _lib = L
    return _lib


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


# ----------------------------------------------------------------------------- tables and scalars

def tables():
    """(palettes [4][4] float64, masks [4] uint32) exactly as the oracle holds them."""
    pal = np.zeros(16, np.float64)
    masks = np.zeros(4, np.uint32)
    lib().oracle_tables(_ptr(pal, ctypes.c_double), _ptr(masks, ctypes.c_uint32))
    return pal.reshape(4, 4), masks


def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def ue8m0_value(E):
    return lib().oracle_ue8m0_value(int(E))


def e5m3_value(b):
    """E5M3 block scale (the reading: no sign, bias 15, subnormals, exponent 31 = NaN)."""
    return lib().oracle_e5m3_value(int(b))


def state_push(s, b):
    return lib().oracle_state_push(int(s), int(b))


def state_decode(s):
    p, e = ctypes.c_int(), ctypes.c_int()
    lib().oracle_state_decode(int(s), ctypes.byref(p), ctypes.byref(e))
    return p.value, e.value


def state_value(s):
    return lib().oracle_state_value(int(s))


def state_code(s):
    return lib().oracle_state_code(int(s))


def bf16_value(bits):
    return lib().oracle_bf16_value(int(bits))


def bf16_round(v):
    return lib().oracle_bf16_round(float(v))


def bf16_bits(v):
    return lib().oracle_bf16_bits(float(v))


def bf16_round_array(a):
    """Elementwise bf16 round-to-nearest-even of a float64 array (returns uint16 bits)."""
    L = lib()
    flat = np.asarray(a, np.float64).ravel()
    out = np.fromiter((L.oracle_bf16_bits(float(v)) for v in flat), np.uint16, flat.size)
    return out.reshape(np.shape(a))


def bf16_bits_to_f64(bits):
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- decode and expand

def _stream_args(stream, scales, rows, cols):
    stream = np.ascontiguousarray(stream, np.uint32)
    if stream.size != rows * (cols // 32) * 2:
        raise ValueError("stream size does not match [rows][cols/32][2]")
    if scales is not None:
        scales = np.ascontiguousarray(scales, np.uint8)
        if scales.size != rows * (cols // 32):
            raise ValueError("scales size does not match [rows][cols/32]")
    return stream, scales


def decode_codes(stream, rows, cols, seg_len):
    stream, _ = _stream_args(stream, None, rows, cols)
    codes = np.zeros((rows, cols), np.uint8)
    _check(lib().oracle_decode_codes(_ptr(stream, ctypes.c_uint32), rows, cols, seg_len,
                                     _ptr(codes, ctypes.c_uint8)), "decode_codes")
    return codes


def decode_values(stream, scales, rows, cols, seg_len, scale_fmt="ue8m0"):
    stream, scales = _stream_args(stream, scales, rows, cols)
    w = np.zeros((rows, cols), np.float64)
    fn = lib().oracle_decode_values_e5m3 if scale_fmt == "e5m3" else lib().oracle_decode_values
    _check(fn(_ptr(stream, ctypes.c_uint32), _ptr(scales, ctypes.c_uint8), rows, cols, seg_len,
              _ptr(w, ctypes.c_double)), "decode_values")
    return w


def decode_codes_interleaved(il, rows, cols, seg_len):
    """Codes [rows][cols] of an interleaved-packed stream, from 16-bit windows of its bit string."""
    il, _ = _stream_args(il, None, rows, cols)
    codes = np.zeros((rows, cols), np.uint8)
    _check(lib().oracle_decode_codes_interleaved(_ptr(il, ctypes.c_uint32), rows, cols, seg_len,
                                                 _ptr(codes, ctypes.c_uint8)), "decode_codes_interleaved")
    return codes


def repack_interleaved(il, rows, cols):
    """Planar stream words [rows][cols/32][2] of an interleaved-packed stream of the same shape."""
    il, _ = _stream_args(il, None, rows, cols)
    out = np.zeros((rows, cols // 32, 2), np.uint32)
    _check(lib().oracle_repack_interleaved(_ptr(il, ctypes.c_uint32), rows, cols, _ptr(out, ctypes.c_uint32)),
           "repack_interleaved")
    return out


def expand_mxfp4(stream, scales, rows, cols, seg_len):
    stream, scales = _stream_args(stream, scales, rows, cols)
    nib = np.zeros((rows, cols // 2), np.uint8)
    sc = np.zeros((rows, cols // 32), np.uint8)
    _check(lib().oracle_expand_mxfp4(_ptr(stream, ctypes.c_uint32), _ptr(scales, ctypes.c_uint8),
                                     rows, cols, seg_len, _ptr(nib, ctypes.c_uint8),
                                     _ptr(sc, ctypes.c_uint8)), "expand_mxfp4")
    return nib, sc


# ----------------------------------------------------------------------------- products

def gemv(stream, scales, rows, cols, seg_len, x_bits, row_ids=None, scale_fmt="ue8m0"):
    """y[T][nr] (fp64) and ||w_row||_2 [nr] for bf16 activations x_bits [T][cols] (uint16);
    scale_fmt "e5m3" reads the scale bytes as E5M3 block scales."""
    stream, scales = _stream_args(stream, scales, rows, cols)
    x_bits = np.ascontiguousarray(np.atleast_2d(x_bits), np.uint16)
    T = x_bits.shape[0]
    if x_bits.shape[1] != cols:
        raise ValueError("x must be [T][cols]")
    if row_ids is None:
        nr, rid = rows, None
    else:
        rid = np.ascontiguousarray(row_ids, np.int64)
        nr = rid.size
    y = np.zeros((T, nr), np.float64)
    wn = np.zeros(nr, np.float64)
    fn = lib().oracle_gemv_e5m3 if scale_fmt == "e5m3" else lib().oracle_gemv
    _check(fn(_ptr(stream, ctypes.c_uint32), _ptr(scales, ctypes.c_uint8), rows, cols, seg_len,
              _ptr(x_bits, ctypes.c_uint16), T, None if rid is None else _ptr(rid, ctypes.c_int64), nr,
              _ptr(y, ctypes.c_double), _ptr(wn, ctypes.c_double)), "gemv")
    return y, wn


def mxfp4_gemv(nibbles, scales, rows, cols, x_bits, row_ids=None):
    """y[T][nr] (fp64) and ||w_row||_2 [nr] from a resident MXFP4 tensor (HEPH mode 2 consumer):
    nibbles uint8 [rows][cols/2], scales uint8 [rows][cols/32], bf16 bits x [T][cols]."""
    nibbles = np.ascontiguousarray(nibbles, np.uint8).reshape(-1)
    scales = np.ascontiguousarray(scales, np.uint8).reshape(-1)
    if nibbles.size != rows * (cols // 2) or scales.size != rows * (cols // 32):
        raise ValueError("nibbles must be [rows][cols/2] and scales [rows][cols/32]")
    x_bits = np.ascontiguousarray(np.atleast_2d(x_bits), np.uint16)
    T = x_bits.shape[0]
    if x_bits.shape[1] != cols:
        raise ValueError("x must be [T][cols]")
    if row_ids is None:
        nr, rid = rows, None
    else:
        rid = np.ascontiguousarray(row_ids, np.int64)
        nr = rid.size
    y = np.zeros((T, nr), np.float64)
    wn = np.zeros(nr, np.float64)
    _check(lib().oracle_mxfp4_gemv(_ptr(nibbles, ctypes.c_uint8), _ptr(scales, ctypes.c_uint8), rows, cols,
                                   _ptr(x_bits, ctypes.c_uint16), T,
                                   None if rid is None else _ptr(rid, ctypes.c_int64), nr,
                                   _ptr(y, ctypes.c_double), _ptr(wn, ctypes.c_double)), "mxfp4_gemv")
    return y, wn


# ----------------------------------------------------------------------------- encoder

def viterbi_encode(target, D, scale):
    """D-weighted Viterbi over one segment ("Curvature-aware Viterbi objective" bullet)."""
    target = np.ascontiguousarray(target, np.float64)
    D = np.ascontiguousarray(D, np.float64)
    scale = np.ascontiguousarray(scale, np.float64)
    L = target.size
    sym = np.zeros(L, np.uint8)
    cost = lib().oracle_viterbi_encode(_ptr(target, ctypes.c_double), _ptr(D, ctypes.c_double),
                                       _ptr(scale, ctypes.c_double), L, _ptr(sym, ctypes.c_uint8))
    if cost < 0:
        raise ValueError("viterbi_encode failed")
    return sym, cost


def bruteforce_encode(target, D, scale):
    target = np.ascontiguousarray(target, np.float64)
    D = np.ascontiguousarray(D, np.float64)
    scale = np.ascontiguousarray(scale, np.float64)
    L = target.size
    sym = np.zeros(L, np.uint8)
    cost = lib().oracle_bruteforce_encode(_ptr(target, ctypes.c_double), _ptr(D, ctypes.c_double),
                                          _ptr(scale, ctypes.c_double), L, _ptr(sym, ctypes.c_uint8))
    if cost < 0:
        raise ValueError("bruteforce_encode takes L <= 8")
    return sym, cost


def pack_symbols(sym, rows, cols):
    """Planar stream words [rows][cols/32][2] holding the branch symbols sym [rows][cols]."""
    sym = np.asarray(sym, np.uint32).reshape(rows, cols // 32, 32)
    bit = np.arange(32, dtype=np.uint32)
    lo = ((sym & 1) << bit).sum(axis=2, dtype=np.uint64).astype(np.uint32)
    hi = (((sym >> 1) & 1) << bit).sum(axis=2, dtype=np.uint64).astype(np.uint32)
    return np.stack([lo, hi], axis=2)


# ----------------------------------------------------------------------------- routing and MoE

def route(logits, k):
    """Top-k experts per token and fp64 softmax over the selected logits.

    Ranking: larger logit first, ties -> lower index; a NaN logit ranks below every number
    (-inf included), so k valid expert ids always come out. Weights: softmax over the k selected
    logits with NaN read as -inf; when the largest selected logit is -inf every weight is 0 (the
    token routes nowhere), and when it is +inf the +inf logits share the weight equally (the limit
    of the softmax)."""
    logits = np.asarray(logits, np.float64)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (bool(np.isnan(logits[t, e])),
                                                0.0 if np.isnan(logits[t, e]) else -logits[t, e], e))[:k]
        sel = np.array([-np.inf if np.isnan(logits[t, e]) else logits[t, e] for e in order])
        ids[t] = order
        mx = sel.max()
        if mx == -np.inf:
            w[t] = 0.0
        elif mx == np.inf:
            w[t] = (sel == np.inf) / np.count_nonzero(sel == np.inf)
        else:
            ex = np.exp(sel - mx)
            w[t] = ex / ex.sum()
    return ids, w


def silu(g):
    g = np.asarray(g, np.float64)
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def _product(layer, kind, e, rows, cols, seg_len, xb):
    """One expert matrix's product: the trellis stream decoded (mode 1) or, when the layer carries
    expanded tensors (attributes gu_nibbles / dn_nibbles), the resident MXFP4 tensor (mode 2)."""
    if hasattr(layer, kind + "_nibbles"):
        return mxfp4_gemv(getattr(layer, kind + "_nibbles")[e], getattr(layer, kind + "_mx_scales")[e], rows, cols, xb)
    return gemv(getattr(layer, kind + "_stream")[e], getattr(layer, kind + "_scales")[e], rows, cols, seg_len, xb)


def moe_hidden(layer, x_bits, ids, seg_len):
    """Exact gate/up products and h = bf16(silu(g) * u) for every (t, j): returns
    g, u [T][k][I] fp64, h_bits [T][k][I] uint16, and the gate/up row norms [T][k][2I]."""
    x_bits = np.atleast_2d(np.asarray(x_bits, np.uint16))
    T, k = ids.shape
    H, I = layer.H, layer.I
    g = np.zeros((T, k, I))
    u = np.zeros((T, k, I))
    norms = np.zeros((T, k, 2 * I))
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            y, wn = _product(layer, "gu", e, 2 * I, H, seg_len, x_bits[t:t + 1])
            g[t, j], u[t, j] = y[0, :I], y[0, I:]
            norms[t, j] = wn
    h_bits = bf16_round_array(silu(g) * u)
    return g, u, h_bits, norms


def moe_down(layer, h_bits, ids, w, seg_len):
    """y_j = down_e . h_j (exact) and out = sum_j w_j y_j in fp64, plus the bound factor
    sum_j |w_j| ||down_row|| ||h_j|| per output. h_bits [T][k][I] bf16 bits."""
    T, k = ids.shape
    H, I = layer.H, layer.I
    out = np.zeros((T, H))
    bound = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            hb = np.asarray(h_bits[t, j], np.uint16)[None, :]
            y, wn = _product(layer, "dn", e, H, I, seg_len, hb)
            hn = np.linalg.norm(bf16_bits_to_f64(hb))
            out[t] += w[t, j] * y[0]
            bound[t] += abs(w[t, j]) * wn * hn
    return out, bound


def moe(layer, x_bits, ids, w, seg_len):
    """The whole layer on the oracle: returns (out fp64 [T][H], h_bits [T][k][I])."""
    _, _, h_bits, _ = moe_hidden(layer, x_bits, ids, seg_len)
    out, _ = moe_down(layer, h_bits, ids, w, seg_len)
    return out, h_bits


def fsum_dot(a, b):
    """Correctly rounded dot product of exact fp64 products (math.fsum)."""
    return math.fsum(float(p) for p in np.asarray(a, np.float64) * np.asarray(b, np.float64))
