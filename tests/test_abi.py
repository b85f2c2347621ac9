"""The C-ABI library loads, exports every symbol include/tcf4.h declares, and rejects bad arguments
on the host before launching anything (these calls make no CUDA call, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

from trellis_coded_fp4_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"TCF4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared()
    assert set(declared) == set(_abi.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(6):
        assert lib.tcf4_status_string(s)
    assert lib.tcf4_status_string(99) == b"unknown status"


def _mat(stream=16, scales=16, rows=4, cols=64, seg=32):
    return _abi.Matrix(stream, scales, rows, cols, seg)


def test_gemv_argument_checks(lib):
    ok_x, ok_y = ctypes.c_void_p(4096), ctypes.c_void_p(8192)
    s0 = ctypes.c_void_p(0)
    ws0 = ctypes.c_void_p(0)

    def gemv(w, x, T, y):  # these checks never reach a launch, so no workspace is involved
        return lib.trellis_gemv(w, x, T, y, ws0, 0, s0)

    assert gemv(_mat(cols=48), ok_x, 1, ok_y) == 1          # cols % 32
    assert gemv(_mat(seg=48), ok_x, 1, ok_y) == 1           # seg_len % 32
    assert gemv(_mat(seg=96), ok_x, 1, ok_y) == 1           # seg_len does not divide cols
    assert gemv(_mat(stream=0), ok_x, 1, ok_y) == 1         # null stream
    assert gemv(_mat(stream=8), ok_x, 1, ok_y) == 2         # misaligned stream
    assert gemv(_mat(), ctypes.c_void_p(4098), 1, ok_y) == 2
    assert gemv(_mat(), ok_x, 33, ok_y) == 3                # T > 32
    assert gemv(_mat(), ok_x, -1, ok_y) == 1
    assert gemv(_mat(), ok_x, 0, ok_y) == 0                 # empty: no launch
    assert gemv(_mat(rows=0), ok_x, 1, ok_y) == 0
    assert gemv(_mat(cols=32768, seg=32), ok_x, 1, ok_y) == 3
    assert gemv(_mat(), ctypes.c_void_p(0), 1, ok_y) == 1


def test_expand_and_route_argument_checks(lib):
    s0 = ctypes.c_void_p(0)
    assert lib.trellis_decode_to_mxfp4(_mat(), ctypes.c_void_p(0), ctypes.c_void_p(64), s0) == 1
    assert lib.trellis_decode_to_mxfp4(_mat(), ctypes.c_void_p(72), ctypes.c_void_p(64), s0) == 2
    assert lib.trellis_decode_to_mxfp4(_mat(rows=0), ctypes.c_void_p(0), ctypes.c_void_p(0), s0) == 0
    p = ctypes.c_void_p(256)
    assert lib.trellis_moe_route(p, 4, 8, 9, p, p, s0) == 1                  # k > E
    assert lib.trellis_moe_route(p, 4, 300, 4, p, p, s0) == 3                # E > 256
    assert lib.trellis_moe_route(p, 4, 32, 9, p, p, s0) == 3                 # k > 8
    assert lib.trellis_moe_route(p, 0, 32, 4, p, p, s0) == 0


def test_moe_workspace_and_checks(lib):
    E, H, I = 4, 64, 96
    gu = (_abi.Matrix * E)(*[_abi.Matrix(256, 256, 2 * I, H, 32) for _ in range(E)])
    dn = (_abi.Matrix * E)(*[_abi.Matrix(256, 256, H, I, 32) for _ in range(E)])
    m = _abi.Moe(gu, dn, E, H, I)
    ws = lib.trellis_grouped_moe_workspace(ctypes.byref(m), 3, 2)
    off = lib.trellis_grouped_moe_hidden_offset(ctypes.byref(m), 3, 2)
    assert ws > 0 and ws % 256 == 0 and 0 < off < ws
    assert ws - off >= 3 * 2 * I * 2 + 3 * 2 * H * 4
    p = ctypes.c_void_p(256)
    s0 = ctypes.c_void_p(0)
    assert lib.trellis_grouped_moe(ctypes.byref(m), p, 3, p, p, 2, p, p, ws - 1, s0) == 4
    assert lib.trellis_grouped_moe(ctypes.byref(m), p, 3, p, p, 2, p, ctypes.c_void_p(0), ws, s0) == 4
    assert lib.trellis_grouped_moe(ctypes.byref(m), p, 3, p, p, 2, p, ctypes.c_void_p(512 + 16), ws, s0) == 2
    assert lib.trellis_grouped_moe(ctypes.byref(m), p, 33, p, p, 2, p, p, ws, s0) == 3
    bad = _abi.Moe(gu, dn, E, H, I + 32)                                      # shapes disagree
    assert lib.trellis_grouped_moe_workspace(ctypes.byref(bad), 3, 2) == 0
    dn2 = (_abi.Matrix * E)(*[_abi.Matrix(256, 256, H, I, 32 if e else 96) for e in range(E)])
    mixed = _abi.Moe(gu, dn2, E, H, I)                                        # mixed seg_len
    assert lib.trellis_grouped_moe(ctypes.byref(mixed), p, 3, p, p, 2, p, p, ws, s0) == 3
    assert lib.trellis_grouped_moe(ctypes.byref(m), p, 0, p, p, 2, p, p, ws, s0) == 0


def test_repack_argument_checks(lib):
    s0 = ctypes.c_void_p(0)
    a, b = ctypes.c_void_p(4096), ctypes.c_void_p(1 << 20)
    rp = lib.trellis_repack_interleaved
    assert rp(a, 2, 48, b, s0) == 1                        # cols % 32
    assert rp(a, -1, 32, b, s0) == 1                       # rows < 0
    assert rp(ctypes.c_void_p(0), 2, 32, b, s0) == 1       # null input
    assert rp(a, 2, 32, ctypes.c_void_p(0), s0) == 1       # null output
    assert rp(ctypes.c_void_p(4100), 2, 32, b, s0) == 2    # 4-byte aligned input
    assert rp(a, 2, 32, ctypes.c_void_p((1 << 20) + 4), s0) == 2
    assert rp(a, 4, 32, ctypes.c_void_p(4096 + 8), s0) == 1   # partial overlap (32 bytes from 4096)
    assert rp(ctypes.c_void_p(4096 + 24), 4, 32, a, s0) == 1  # overlap from the other side
    assert rp(a, 1 << 31, 32 * 2, b, s0) == 3              # 2^32 blocks
    assert rp(a, 0, 32, b, s0) == 0 and rp(a, 3, 0, b, s0) == 0   # nothing to do


def test_e5m3_gemv_argument_checks(lib):
    s0 = ctypes.c_void_p(0)
    ok_x, ok_y = ctypes.c_void_p(4096), ctypes.c_void_p(8192)
    ws0 = ctypes.c_void_p(0)

    def g(w, x, T, y, s):  # these checks never reach a launch, so no workspace is involved
        return lib.trellis_gemv_e5m3(w, x, T, y, ws0, 0, s)

    assert g(_mat(cols=48), ok_x, 1, ok_y, s0) == 1
    assert g(_mat(seg=96), ok_x, 1, ok_y, s0) == 1
    assert g(_mat(stream=8), ok_x, 1, ok_y, s0) == 2
    assert g(_mat(), ctypes.c_void_p(4098), 1, ok_y, s0) == 2
    assert g(_mat(), ok_x, 1, ctypes.c_void_p(8200), s0) == 2
    assert g(_mat(), ok_x, 33, ok_y, s0) == 3
    assert g(_mat(), ok_x, -1, ok_y, s0) == 1
    assert g(_mat(), ctypes.c_void_p(0), 1, ok_y, s0) == 1
    assert g(_mat(), ok_x, 0, ok_y, s0) == 0 and g(_mat(rows=0), ok_x, 1, ok_y, s0) == 0
    assert lib.trellis_gemv_e5m3_workspace(_mat(cols=48), 1) == 0


def test_e5m3_scale_sets_sum_to_the_e5m3_value():
    # The tensor-core path writes each E5M3 scale as four powers of two (UE8M0 bytes, byte 0 read as
    # 2^-127 and standing for an absent power): restated here, their sum must be the oracle's E5M3
    # value for every byte, up to the 2^-127 stand-ins; byte 0xF8.. (NaN) gives a NaN byte.
    import oracle
    for b in range(256):
        e, m = b >> 3, b & 7
        nz, nan, ee = int(e >= 1), int(e == 31), max(e, 1)
        st = [((e + 112) if nz else 0) | (0xFF if nan else 0),
              (ee + 111) if (m >> 2) & 1 else 0, (ee + 110) if (m >> 1) & 1 else 0, (ee + 109) if m & 1 else 0]
        if nan:
            assert st[0] == 0xFF
            continue
        total = sum(2.0 ** (v - 127) for v in st if v != 0)
        tiny = sum(1 for v in st if v == 0) * 2.0 ** -127
        assert total == oracle.e5m3_value(b), b
        assert all(0 <= v < 255 for v in st) and tiny <= 4 * 2.0 ** -127


def test_encode_argument_checks(lib):
    s0 = ctypes.c_void_p(0)
    p8, p16 = ctypes.c_void_p(8 * 512), ctypes.c_void_p(16 * 512)
    ws = ctypes.c_void_p(256 * 64)
    e = lib.trellis_encode
    assert e(p8, p8, p16, 2, 64, 48, p8, s0, ws, 1 << 20, s0) == 1    # seg % 32
    assert e(p8, p8, p16, 2, 64, 128, p8, s0, ws, 1 << 20, s0) == 1   # seg > cols
    assert e(p8, p8, p16, 2, 48, 32, p8, s0, ws, 1 << 20, s0) == 1    # cols % 32
    assert e(ctypes.c_void_p(8 * 512 + 4), p8, p16, 2, 64, 32, p8, s0, ws, 1 << 20, s0) == 2
    assert e(p8, p8, p16, 2, 64, 32, p8, s0, s0, 0, s0) == 4          # no workspace
    assert e(p8, p8, p16, 2, 64, 32, p8, s0, ctypes.c_void_p(256 * 64 + 128), 1 << 20, s0) == 2
    assert e(p8, p8, p16, 1 << 20, 1 << 12, 32, p8, s0, ws, 1 << 20, s0) == 3   # 2^32 weights
    assert e(p8, p8, p16, 0, 64, 32, p8, s0, s0, 0, s0) == 0


def test_scale_tile_sizes_and_checks(lib):
    # 128-row tiles x 8 groups per started 1024 columns x 512 bytes; host checks before any launch
    assert lib.trellis_scale_tiles_bytes(_mat(rows=1, cols=64)) == 1 * 8 * 512
    assert lib.trellis_scale_tiles_bytes(_mat(rows=128, cols=1024)) == 1 * 8 * 512
    assert lib.trellis_scale_tiles_bytes(_mat(rows=129, cols=1056)) == 2 * 16 * 512
    assert lib.trellis_scale_tiles_bytes(_mat(rows=184320, cols=2880)) == 1440 * 24 * 512
    assert lib.trellis_scale_tiles_bytes(_mat(rows=0)) == 0
    assert lib.trellis_scale_tiles_bytes(_mat(cols=48)) == 0
    s0 = ctypes.c_void_p(0)
    assert lib.trellis_make_scale_tiles(_mat(), ctypes.c_void_p(0), s0) == 1       # null tiles
    assert lib.trellis_make_scale_tiles(_mat(), ctypes.c_void_p(4104), s0) == 2    # misaligned tiles
    assert lib.trellis_make_scale_tiles(_mat(cols=48), ctypes.c_void_p(4096), s0) == 1
    assert lib.trellis_make_scale_tiles(_mat(rows=0), ctypes.c_void_p(0), s0) == 0  # empty: nothing to do
    ok_x, ok_y, ok_t = ctypes.c_void_p(4096), ctypes.c_void_p(8192), ctypes.c_void_p(16384)

    def gemv_tiled(w, t, x, T, y):
        return lib.trellis_gemv_tiled(w, t, x, T, y, ctypes.c_void_p(0), 0, s0)

    assert gemv_tiled(_mat(scales=0), ctypes.c_void_p(0), ok_x, 1, ok_y) == 1   # null tiles
    assert gemv_tiled(_mat(scales=0), ctypes.c_void_p(16392), ok_x, 1, ok_y) == 2
    assert gemv_tiled(_mat(), ok_t, ok_x, 33, ok_y) == 3                         # T > 32
    assert gemv_tiled(_mat(cols=48), ok_t, ok_x, 1, ok_y) == 1
    assert gemv_tiled(_mat(), ok_t, ok_x, 0, ok_y) == 0                          # T == 0: no-op
