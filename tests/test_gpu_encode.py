"""GPU parity for the D-weighted Viterbi encoder (trellis_encode) against the oracle's encoder.

The XOR-Trellis page's "Curvature-aware Viterbi objective" bullet defines the search; the oracle
(pinned against exhaustive search) gives, per segment, the symbols and the minimum cost. Both sides
evaluate the objective in fp64 term by term with no fused operations, and break ties the same way,
so the symbols (stream words) and the costs must match exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import _abi, synth

pytestmark = pytest.mark.gpu


def _inputs(rows, cols, seed, lo=120, hi=128):
    r = np.random.default_rng(seed)
    sc = r.integers(lo, hi, size=(rows, cols // 32), dtype=np.uint8)
    scale = np.repeat(2.0 ** (sc.astype(np.float64) - 127), 32, axis=1)
    target = r.normal(0, 2.5, (rows, cols)) * scale
    D = r.uniform(0.1, 10.0, (rows, cols))
    return target, D, sc, scale


def _gpu_encode(target, D, sc, seg, ws_bytes=None):
    rows, cols = target.shape
    t = torch.from_numpy(target).cuda()
    d = torch.from_numpy(D).cuda()
    s = torch.from_numpy(sc.reshape(-1)).cuda()
    ws = None
    if ws_bytes is not None:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    W, cost = tc.encode(t, d, s, seg, workspace=ws)
    torch.cuda.synchronize()
    stream = W.stream.cpu().numpy().view(np.uint32).reshape(rows, cols // 32, 2)
    return stream, cost.cpu().numpy()


def _oracle_encode(target, D, scale, seg):
    rows, cols = target.shape
    sym = np.zeros((rows, cols), np.uint8)
    cost = np.zeros((rows, cols // seg))
    for n in range(rows):
        for j in range(cols // seg):
            sl = slice(j * seg, (j + 1) * seg)
            sym[n, sl], cost[n, j] = oracle.viterbi_encode(target[n, sl], D[n, sl], scale[n, sl])
    return oracle.pack_symbols(sym, rows, cols), cost


@pytest.mark.parametrize("seg", [32, 64, 128])
def test_encode_matches_oracle_exactly(seg):
    rows, cols = 3, 128
    target, D, sc, scale = _inputs(rows, cols, 9000 + seg)
    st_g, c_g = _gpu_encode(target, D, sc, seg)
    st_o, c_o = _oracle_encode(target, D, scale, seg)
    assert np.array_equal(c_g, c_o), f"costs differ: {c_g} vs {c_o}"
    assert np.array_equal(st_g, st_o)


def test_encode_ties_follow_the_same_rule():
    # a zero target makes every path cost the same wherever the decoded values are +-0: equal-cost
    # paths everywhere, so only the tie rule decides
    rows, cols, seg = 2, 64, 32
    _, D, sc, scale = _inputs(rows, cols, 9100)
    target = np.zeros((rows, cols))
    D = np.ones((rows, cols))
    st_g, c_g = _gpu_encode(target, D, sc, seg)
    st_o, c_o = _oracle_encode(target, D, scale, seg)
    assert np.array_equal(c_g, c_o) and np.array_equal(st_g, st_o)


@pytest.mark.parametrize("seg", [32, 256])
def test_encode_of_decoded_stream_round_trips(seg):
    # decoded values are reachable exactly, and the decoder is one-to-one on a segment: the encoder
    # must return the stream itself at cost 0
    rows, cols = 4, 256
    st = synth.stream(rows, cols, 9200 + seg)
    sc = synth.scales(rows, cols, 9200 + seg)
    w = oracle.decode_values(st, sc, rows, cols, seg)
    D = np.random.default_rng(seg).uniform(0.01, 5.0, (rows, cols))
    st_g, c_g = _gpu_encode(w, D, sc, seg)
    assert np.array_equal(c_g, np.zeros_like(c_g))
    assert np.array_equal(st_g, st)


def test_encode_with_one_segment_at_a_time():
    # a workspace for a single CTA runs the segments one after another, with the same result
    rows, cols, seg = 2, 96, 32
    target, D, sc, scale = _inputs(rows, cols, 9300)
    st_g, c_g = _gpu_encode(target, D, sc, seg, ws_bytes=seg * 4096)
    st_o, c_o = _oracle_encode(target, D, scale, seg)
    assert np.array_equal(c_g, c_o) and np.array_equal(st_g, st_o)


def test_encode_argument_errors():
    L = _abi.load()
    t = torch.zeros((2, 64), dtype=torch.float64, device="cuda")
    s = torch.full((2 * 2,), 127, dtype=torch.uint8, device="cuda")
    out = torch.empty(2 * 2 * 2, dtype=torch.int32, device="cuda")
    ws = torch.empty(tc.encode_workspace_bytes(2, 64, 32), dtype=torch.uint8, device="cuda")
    p = lambda x: x.data_ptr()
    assert L.trellis_encode(p(t), p(t), p(s), 2, 64, 48, p(out), None, p(ws), ws.numel(), None) == 1   # seg % 32
    assert L.trellis_encode(p(t), p(t), p(s), 2, 64, 128, p(out), None, p(ws), ws.numel(), None) == 1  # seg > cols
    assert L.trellis_encode(p(t), p(t), p(s), 2, 64, 32, p(out), None, p(ws), 1000, None) == 4
    assert L.trellis_encode(p(t) + 4, p(t), p(s), 2, 64, 32, p(out), None, p(ws), ws.numel(), None) == 2
    assert L.trellis_encode(p(t), p(t), p(s), 0, 64, 32, p(out), None, None, 0, None) == 0
    torch.cuda.synchronize()


def test_encode_no_bounded_wait_gave_up():
    assert tc.device_timeouts() == 0
