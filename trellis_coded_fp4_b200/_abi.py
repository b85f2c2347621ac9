"""ctypes declarations for the C ABI in include/tcf4.h (argument marshalling only)."""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtcf4.so")

TCF4_OK = 0
STATUS_NAMES = {0: "TCF4_OK", 1: "TCF4_ERR_INVALID_ARG", 2: "TCF4_ERR_MISALIGNED", 3: "TCF4_ERR_UNSUPPORTED",
                4: "TCF4_ERR_WORKSPACE", 5: "TCF4_ERR_CUDA"}

# Every symbol include/tcf4.h declares.
EXPORTED = ("trellis_decode_to_mxfp4", "trellis_gemv_workspace", "trellis_gemv", "trellis_gemv_noalloc",
            "trellis_moe_route", "trellis_grouped_moe_workspace",
            "trellis_grouped_moe", "trellis_grouped_moe_hidden_offset", "mxfp4_gemv_workspace", "mxfp4_gemv",
            "mxfp4_grouped_moe_workspace", "mxfp4_grouped_moe_hidden_offset", "mxfp4_grouped_moe",
            "trellis_encode_workspace", "trellis_encode", "trellis_repack_interleaved", "trellis_gemv_e5m3",
            "trellis_gemv_e5m3_workspace",
            "trellis_scale_tiles_bytes", "trellis_make_scale_tiles", "trellis_gemv_tiled",
            "tcf4_device_timeouts", "tcf4_status_string")


class Matrix(ctypes.Structure):
    """tcf4_matrix"""
    _fields_ = [("stream", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("seg_len", ctypes.c_int32)]


class Moe(ctypes.Structure):
    """tcf4_moe"""
    _fields_ = [("gate_up", ctypes.POINTER(Matrix)), ("down", ctypes.POINTER(Matrix)), ("E", ctypes.c_int32),
                ("H", ctypes.c_int32), ("I", ctypes.c_int32)]


class Mxfp4(ctypes.Structure):
    """tcf4_mxfp4"""
    _fields_ = [("nibbles", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64)]


class Mxfp4Moe(ctypes.Structure):
    """tcf4_mxfp4_moe"""
    _fields_ = [("gate_up", ctypes.POINTER(Mxfp4)), ("down", ctypes.POINTER(Mxfp4)), ("E", ctypes.c_int32),
                ("H", ctypes.c_int32), ("I", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libtcf4.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libtcf4.so not found at {path}; build it with "
                           "`python -m trellis_coded_fp4_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    L.trellis_decode_to_mxfp4.argtypes = [Matrix, vp, vp, vp]
    L.trellis_decode_to_mxfp4.restype = ctypes.c_int
    L.trellis_repack_interleaved.argtypes = [vp, ctypes.c_int64, ctypes.c_int64, vp, vp]
    L.trellis_gemv_e5m3_workspace.argtypes = [Matrix, ctypes.c_int32]
    L.trellis_gemv_e5m3_workspace.restype = ctypes.c_size_t
    L.trellis_gemv_e5m3.argtypes = [Matrix, vp, ctypes.c_int32, vp, vp, ctypes.c_size_t, vp]
    L.trellis_gemv_e5m3.restype = ctypes.c_int
    L.trellis_repack_interleaved.restype = ctypes.c_int
    L.trellis_gemv_workspace.argtypes = [Matrix, i32]
    L.trellis_gemv_workspace.restype = sz
    L.trellis_gemv.argtypes = [Matrix, vp, i32, vp, vp, sz, vp]
    L.trellis_gemv.restype = ctypes.c_int
    L.trellis_scale_tiles_bytes.argtypes = [Matrix]
    L.trellis_scale_tiles_bytes.restype = sz
    L.trellis_make_scale_tiles.argtypes = [Matrix, vp, vp]
    L.trellis_make_scale_tiles.restype = ctypes.c_int
    L.trellis_gemv_tiled.argtypes = [Matrix, vp, vp, i32, vp, vp, sz, vp]
    L.trellis_gemv_tiled.restype = ctypes.c_int
    L.trellis_gemv_noalloc.argtypes = [Matrix, vp, i32, vp, vp]
    L.trellis_gemv_noalloc.restype = ctypes.c_int
    L.trellis_moe_route.argtypes = [vp, i32, i32, i32, vp, vp, vp]
    L.trellis_moe_route.restype = ctypes.c_int
    L.trellis_grouped_moe_workspace.argtypes = [ctypes.POINTER(Moe), i32, i32]
    L.trellis_grouped_moe_workspace.restype = sz
    L.trellis_grouped_moe_hidden_offset.argtypes = [ctypes.POINTER(Moe), i32, i32]
    L.trellis_grouped_moe_hidden_offset.restype = sz
    L.trellis_grouped_moe.argtypes = [ctypes.POINTER(Moe), vp, i32, vp, vp, i32, vp, vp, sz, vp]
    L.trellis_grouped_moe.restype = ctypes.c_int
    L.mxfp4_gemv_workspace.argtypes = [Mxfp4, i32]
    L.mxfp4_gemv_workspace.restype = sz
    L.mxfp4_gemv.argtypes = [Mxfp4, vp, i32, vp, vp, sz, vp]
    L.mxfp4_gemv.restype = ctypes.c_int
    L.mxfp4_grouped_moe_workspace.argtypes = [ctypes.POINTER(Mxfp4Moe), i32, i32]
    L.mxfp4_grouped_moe_workspace.restype = sz
    L.mxfp4_grouped_moe_hidden_offset.argtypes = [ctypes.POINTER(Mxfp4Moe), i32, i32]
    L.mxfp4_grouped_moe_hidden_offset.restype = sz
    L.mxfp4_grouped_moe.argtypes = [ctypes.POINTER(Mxfp4Moe), vp, i32, vp, vp, i32, vp, vp, sz, vp]
    L.mxfp4_grouped_moe.restype = ctypes.c_int
    L.trellis_encode_workspace.argtypes = [i64, i64, i32]
    L.trellis_encode_workspace.restype = sz
    L.trellis_encode.argtypes = [vp, vp, vp, i64, i64, i32, vp, vp, vp, sz, vp]
    L.trellis_encode.restype = ctypes.c_int
    L.tcf4_device_timeouts.argtypes = []
    L.tcf4_device_timeouts.restype = ctypes.c_uint
    L.tcf4_status_string.argtypes = [ctypes.c_int]
    L.tcf4_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


class Tcf4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = load().tcf4_status_string(status).decode()
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({msg})")


def check(status: int, what: str):
    if status != TCF4_OK:
        raise Tcf4Error(status, what)
