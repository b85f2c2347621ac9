"""GPU parity for trellis_repack_interleaved (interleaved stream packing -> planar words).

The oracle repacks by the packing's definition and, separately, decodes an interleaved stream from
16-bit windows of its bit string (the XOR-Trellis page's "16-bit sliding state"). Repacking is
integer work: every output word must match bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import _abi, synth

pytestmark = pytest.mark.gpu


def _il(rows, cols, seed):
    return np.random.default_rng(seed).integers(0, 2**32, size=(rows, cols // 32, 2), dtype=np.uint32)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


def _host(t):
    return t.cpu().numpy().view(np.uint32)


# nblocks = 3, 15, 630, 11700, 2049: ragged tails of every length against four-block units, one and
# several CTAs (a CTA covers 2048 blocks with 32-byte accesses)
SHAPES = [(3, 32), (5, 96), (7, 2880), (130, 2880), (2049, 32)]


@pytest.mark.parametrize("rows,cols", SHAPES)
def test_repack_bit_exact(rows, cols):
    il = _il(rows, cols, 40 + rows)
    out = tc.repack_interleaved(_dev(il), rows, cols)
    torch.cuda.synchronize()
    assert np.array_equal(_host(out).reshape(rows, cols // 32, 2), oracle.repack_interleaved(il, rows, cols))


@pytest.mark.parametrize("in_off,out_off", [(0, 0), (8, 8), (16, 16), (0, 8), (16, 0), (24, 8)])
def test_repack_alignments(in_off, out_off):
    # byte offsets from 256-byte aligned bases: both 32-byte aligned -> 4 blocks per access; both
    # 16-byte aligned -> 2; otherwise 1. Bytes around the output stay untouched.
    rows, cols = 11, 352  # 121 blocks
    il = _il(rows, cols, 300 + in_off + out_off)
    n = il.size
    src = torch.zeros(n + 16, dtype=torch.int32, device="cuda")
    dst = torch.full((n + 16,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    assert src.data_ptr() % 256 == 0 and dst.data_ptr() % 256 == 0
    src[in_off // 4:in_off // 4 + n] = _dev(il.reshape(-1))
    out = dst[out_off // 4:out_off // 4 + n]
    tc.repack_interleaved(src[in_off // 4:in_off // 4 + n], rows, cols, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(_host(out).reshape(rows, cols // 32, 2), oracle.repack_interleaved(il, rows, cols))
    d = _host(dst)
    assert (d[:out_off // 4] == 0x5A5A5A5A).all() and (d[out_off // 4 + n:] == 0x5A5A5A5A).all()


@pytest.mark.parametrize("off", [0, 8, 16])
def test_repack_in_place(off):
    rows, cols = 9, 2880
    il = _il(rows, cols, 500 + off)
    buf = torch.zeros(il.size + 8, dtype=torch.int32, device="cuda")
    view = buf[off // 4:off // 4 + il.size]
    view.copy_(_dev(il.reshape(-1)))
    tc.repack_interleaved(view, rows, cols, out=view)
    torch.cuda.synchronize()
    assert np.array_equal(_host(view).reshape(rows, cols // 32, 2), oracle.repack_interleaved(il, rows, cols))


@pytest.mark.parametrize("seg", [32, 2880])
def test_repacked_stream_decodes_like_the_window_reading(seg):
    # end to end: repack, then expand to MXFP4 on the GPU; every code must be the one the oracle
    # reads from 16-bit windows of the interleaved bit string
    rows, cols = 6, 2880
    il = _il(rows, cols, 700 + seg)
    sc = synth.scales(rows, cols, 700 + seg)
    planar = tc.repack_interleaved(_dev(il), rows, cols)
    W = tc.TrellisMatrix(planar.reshape(-1), torch.from_numpy(sc.reshape(-1)).cuda(), rows, cols, seg)
    nib, _ = tc.decode_to_mxfp4(W)
    torch.cuda.synchronize()
    codes = oracle.decode_codes_interleaved(il, rows, cols, seg)
    want = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    assert np.array_equal(nib.cpu().numpy(), want)


def test_repack_full_size_sampled():
    # a 184320 x 2880 stream (16.6 M blocks, 133 MB; the gate/up matrices of the 32-expert hidden-2880
    # layer stacked), in the launch configuration the bench times; sampled rows checked bit-exactly
    rows, cols = 32 * 5760, 2880
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    il = torch.randint(-2**31, 2**31 - 1, (rows, cols // 32, 2), dtype=torch.int32, device="cuda", generator=g)
    out = tc.repack_interleaved(il, rows, cols)
    torch.cuda.synchronize()
    sample = np.concatenate([[0, rows - 1], np.random.default_rng(3).choice(rows, 62, replace=False)])
    idx = torch.from_numpy(sample).cuda()
    src = _host(il[idx]).reshape(len(sample), cols // 32, 2)
    assert np.array_equal(_host(out[idx]).reshape(len(sample), cols // 32, 2),
                          oracle.repack_interleaved(src, len(sample), cols))


def test_repack_argument_errors():
    L = _abi.load()
    a = torch.zeros(64, dtype=torch.int32, device="cuda")
    b = torch.zeros(64, dtype=torch.int32, device="cuda")
    p = lambda t, off=0: t.data_ptr() + off
    assert L.trellis_repack_interleaved(p(a), 2, 48, p(b), None) == 1      # cols % 32
    assert L.trellis_repack_interleaved(p(a), -1, 32, p(b), None) == 1     # rows < 0
    assert L.trellis_repack_interleaved(None, 2, 32, p(b), None) == 1      # null input
    assert L.trellis_repack_interleaved(p(a, 4), 2, 32, p(b), None) == 2   # 4-byte aligned input
    assert L.trellis_repack_interleaved(p(a), 2, 32, p(b, 12), None) == 2  # 4-byte aligned output
    assert L.trellis_repack_interleaved(p(a), 4, 32, p(a, 8), None) == 1   # partial overlap
    assert L.trellis_repack_interleaved(p(a), 0, 32, p(b), None) == 0      # nothing to do
    assert L.trellis_repack_interleaved(None, 0, 0, None, None) == 0
    torch.cuda.synchronize()
