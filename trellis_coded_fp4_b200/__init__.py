"""Trellis-coded FP4 (XOR-Trellis / HEPH) decode kernels for B200 — Python binding.

Thin wrappers over the C ABI of ``libtcf4.so`` (include/tcf4.h): they take torch CUDA tensors,
pass their device pointers and the current CUDA stream, and raise on a non-OK status. Every step
of the computation runs in the library's sm_100a kernels; there is no CPU fallback. PyTorch only
provides device memory and streams.

Serving modes ("HEPH: 3-Bit Grid-Aligned Trellis Quantization of MXFP4 Mixture-of-Experts ..."):
* mode 1 — the compressed stream stays resident and is decoded inside the product:
  :func:`gemv`, :func:`grouped_moe` (with :func:`moe_route`);
* mode 2 — the stream is expanded once into a resident packed MXFP4 tensor: :func:`decode_to_mxfp4`.
"""
import ctypes

import torch

from . import _abi

__all__ = ["TrellisMatrix", "MoEWeights", "decode_to_mxfp4", "gemv", "gemv_workspace_bytes", "scale_tiles",
           "gemv_tiled", "moe_route",
           "grouped_moe",
           "moe_workspace_bytes", "moe_hidden_offset", "device_timeouts", "Tcf4Error"]

Tcf4Error = _abi.Tcf4Error


def _stream_handle():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


class TrellisMatrix:
    """A resident trellis-coded matrix W [rows][cols]: stream words [rows][cols/32][2] (32-bit,
    kept as an int32 tensor) and UE8M0 scales [rows][cols/32] (uint8), both on the GPU."""

    def __init__(self, stream: torch.Tensor, scales: torch.Tensor, rows: int, cols: int, seg_len: int = 32):
        self.stream, self.scales = stream, scales
        self.rows, self.cols, self.seg_len = int(rows), int(cols), int(seg_len)

    @classmethod
    def from_numpy(cls, stream_np, scales_np, rows, cols, seg_len=32, device="cuda"):
        st = torch.from_numpy(stream_np.view("int32").reshape(-1)).to(device)
        sc = torch.from_numpy(scales_np.reshape(-1)).to(device)
        return cls(st, sc, rows, cols, seg_len)

    def abi(self) -> _abi.Matrix:
        return _abi.Matrix(self.stream.data_ptr(), self.scales.data_ptr(), self.rows, self.cols, self.seg_len)


def decode_to_mxfp4(w: TrellisMatrix, out_nibbles=None, out_scales=None):
    """Expand to packed MXFP4: (nibbles uint8 [rows][cols/2], scales uint8 [rows][cols/32])."""
    dev = w.stream.device
    if out_nibbles is None:
        out_nibbles = torch.empty((w.rows, w.cols // 2), dtype=torch.uint8, device=dev)
    if out_scales is None:
        out_scales = torch.empty((w.rows, w.cols // 32), dtype=torch.uint8, device=dev)
    _abi.check(_abi.load().trellis_decode_to_mxfp4(w.abi(), _ptr(out_nibbles), _ptr(out_scales), _stream_handle()),
               "trellis_decode_to_mxfp4")
    return out_nibbles, out_scales


def repack_interleaved(stream: torch.Tensor, rows: int, cols: int, out=None):
    """Interleaved-packed stream words (each row one bit string, two bits per symbol, low bit first)
    -> the planar words TrellisMatrix holds; int32 [rows][cols/32][2]. out=stream converts in place."""
    if out is None:
        out = torch.empty((rows, cols // 32, 2), dtype=torch.int32, device=stream.device)
    _abi.check(_abi.load().trellis_repack_interleaved(_ptr(stream), rows, cols, _ptr(out), _stream_handle()),
               "trellis_repack_interleaved")
    return out


def gemv_workspace_bytes(w: TrellisMatrix, T: int) -> int:
    """Scratch bytes trellis_gemv needs for T tokens (0: the call needs none)."""
    return int(_abi.load().trellis_gemv_workspace(w.abi(), T))


def gemv(w: TrellisMatrix, x: torch.Tensor, out=None, workspace=None):
    """y = bf16(W x) for bf16 activations x [T][cols] (T <= 32): returns bf16 [T][rows]."""
    x = x if x.dim() == 2 else x.view(1, -1)
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, w.rows), dtype=torch.bfloat16, device=x.device)
    need = gemv_workspace_bytes(w, T)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    nbytes = workspace.numel() if workspace is not None else 0
    _abi.check(_abi.load().trellis_gemv(w.abi(), _ptr(x), T, _ptr(out), _ptr(workspace), nbytes, _stream_handle()),
               "trellis_gemv")
    return out


def scale_tiles_bytes(w: TrellisMatrix) -> int:
    """Bytes of w's scale tiles (trellis_scale_tiles_bytes)."""
    return int(_abi.load().trellis_scale_tiles_bytes(w.abi()))


def scale_tiles(w: TrellisMatrix, out=None):
    """The weights' UE8M0 scales rearranged once into scale tiles (uint8, trellis_scale_tiles_bytes
    long), the layout trellis_gemv_tiled reads."""
    n = scale_tiles_bytes(w)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=w.stream.device)
    _abi.check(_abi.load().trellis_make_scale_tiles(w.abi(), _ptr(out), _stream_handle()), "trellis_make_scale_tiles")
    return out


def gemv_tiled(w: TrellisMatrix, tiles: torch.Tensor, x: torch.Tensor, out=None, workspace=None):
    """gemv with the weights' scales read from scale tiles (see scale_tiles): bf16 [T][rows]."""
    x = x if x.dim() == 2 else x.view(1, -1)
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, w.rows), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(gemv_workspace_bytes(w, T), 1), dtype=torch.uint8, device=x.device)
    _abi.check(_abi.load().trellis_gemv_tiled(w.abi(), _ptr(tiles), _ptr(x), T, _ptr(out), _ptr(workspace),
                                              workspace.numel(), _stream_handle()), "trellis_gemv_tiled")
    return out


def gemv_e5m3_workspace_bytes(w: TrellisMatrix, T: int) -> int:
    """Scratch bytes trellis_gemv_e5m3 needs for T tokens (0: the call needs none)."""
    return int(_abi.load().trellis_gemv_e5m3_workspace(w.abi(), T))


def gemv_e5m3(w: TrellisMatrix, x: torch.Tensor, out=None, workspace=None):
    """y = bf16(W x) with w.scales read as E5M3 block scales: bf16 [T][rows]."""
    x = x if x.dim() == 2 else x.view(1, -1)
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, w.rows), dtype=torch.bfloat16, device=x.device)
    need = gemv_e5m3_workspace_bytes(w, T)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    nbytes = workspace.numel() if workspace is not None else 0
    _abi.check(_abi.load().trellis_gemv_e5m3(w.abi(), _ptr(x), T, _ptr(out), _ptr(workspace), nbytes,
                                             _stream_handle()), "trellis_gemv_e5m3")
    return out


def gemv_noalloc(w: TrellisMatrix, x: torch.Tensor, out=None):
    """gemv through trellis_gemv_noalloc: the scratch is the library's own per-device array."""
    x = x if x.dim() == 2 else x.view(1, -1)
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, w.rows), dtype=torch.bfloat16, device=x.device)
    _abi.check(_abi.load().trellis_gemv_noalloc(w.abi(), _ptr(x), T, _ptr(out), _stream_handle()),
               "trellis_gemv_noalloc")
    return out


def moe_route(logits: torch.Tensor, k: int, ids=None, wts=None):
    """Top-k experts (ties to the lower index) and softmax weights over the selected logits."""
    T, E = logits.shape
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if wts is None:
        wts = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _abi.check(_abi.load().trellis_moe_route(_ptr(logits), T, E, k, _ptr(ids), _ptr(wts), _stream_handle()),
               "trellis_moe_route")
    return ids, wts


class MoEWeights:
    """E experts of one MoE layer: gate_up [2I][H] and down [H][I] trellis matrices per expert."""

    def __init__(self, gate_up, down, H: int, I: int):
        assert len(gate_up) == len(down)
        self.gate_up, self.down = list(gate_up), list(down)
        self.E, self.H, self.I = len(gate_up), int(H), int(I)
        self._gu = (_abi.Matrix * self.E)(*[m.abi() for m in self.gate_up])
        self._dn = (_abi.Matrix * self.E)(*[m.abi() for m in self.down])
        self._moe = _abi.Moe(self._gu, self._dn, self.E, self.H, self.I)

    @classmethod
    def from_layer(cls, layer, seg_len=32, seg_len_down=None, device="cuda"):
        """Upload a synth.MoELayer: one contiguous buffer per kind, one view per expert.
        seg_len applies to gate_up (cols H), seg_len_down (default: seg_len) to down (cols I)."""
        seg_dn = seg_len if seg_len_down is None else seg_len_down
        E, H, I = layer.E, layer.H, layer.I
        gu = torch.from_numpy(layer.gu_stream.view("int32").reshape(E, -1)).to(device)
        gus = torch.from_numpy(layer.gu_scales.reshape(E, -1)).to(device)
        dn = torch.from_numpy(layer.dn_stream.view("int32").reshape(E, -1)).to(device)
        dns = torch.from_numpy(layer.dn_scales.reshape(E, -1)).to(device)
        obj = cls([TrellisMatrix(gu[e], gus[e], 2 * I, H, seg_len) for e in range(E)],
                  [TrellisMatrix(dn[e], dns[e], H, I, seg_dn) for e in range(E)], H, I)
        obj._storage = (gu, gus, dn, dns)
        return obj

    def workspace_bytes(self, T: int, k: int) -> int:
        return int(_abi.load().trellis_grouped_moe_workspace(ctypes.byref(self._moe), T, k))

    def hidden_offset(self, T: int, k: int) -> int:
        return int(_abi.load().trellis_grouped_moe_hidden_offset(ctypes.byref(self._moe), T, k))


class Mxfp4Matrix:
    """A resident MXFP4 matrix W [rows][cols]: nibbles uint8 [rows][cols/2] (element 2u in the low
    nibble of byte u) and UE8M0 scales uint8 [rows][cols/32], both on the GPU (the output of
    decode_to_mxfp4)."""

    def __init__(self, nibbles: torch.Tensor, scales: torch.Tensor, rows: int, cols: int):
        self.nibbles, self.scales = nibbles, scales
        self.rows, self.cols = int(rows), int(cols)

    @classmethod
    def expand(cls, w: "TrellisMatrix"):
        """Expand a trellis matrix once into a resident MXFP4 tensor."""
        nib, sc = decode_to_mxfp4(w)
        return cls(nib, sc, w.rows, w.cols)

    def abi(self) -> _abi.Mxfp4:
        return _abi.Mxfp4(self.nibbles.data_ptr(), self.scales.data_ptr(), self.rows, self.cols)


def mxfp4_gemv_workspace_bytes(w: Mxfp4Matrix, T: int) -> int:
    return int(_abi.load().mxfp4_gemv_workspace(w.abi(), T))


def mxfp4_gemv(w: Mxfp4Matrix, x: torch.Tensor, out=None, workspace=None):
    """y = bf16(W x) from the resident MXFP4 tensor, bf16 activations x [T][cols] (T <= 32)."""
    x = x if x.dim() == 2 else x.view(1, -1)
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, w.rows), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(mxfp4_gemv_workspace_bytes(w, T), 1), dtype=torch.uint8, device=x.device)
    _abi.check(_abi.load().mxfp4_gemv(w.abi(), _ptr(x), T, _ptr(out), _ptr(workspace), workspace.numel(),
                                      _stream_handle()), "mxfp4_gemv")
    return out


class Mxfp4MoEWeights:
    """E experts of one MoE layer as resident MXFP4: gate_up [2I][H] and down [H][I] per expert."""

    def __init__(self, gate_up, down, H: int, I: int):
        assert len(gate_up) == len(down)
        self.gate_up, self.down = list(gate_up), list(down)
        self.E, self.H, self.I = len(gate_up), int(H), int(I)
        self._gu = (_abi.Mxfp4 * self.E)(*[m.abi() for m in self.gate_up])
        self._dn = (_abi.Mxfp4 * self.E)(*[m.abi() for m in self.down])
        self._moe = _abi.Mxfp4Moe(self._gu, self._dn, self.E, self.H, self.I)

    @classmethod
    def expand(cls, m: "MoEWeights"):
        """Expand every expert of a trellis MoE layer once."""
        return cls([Mxfp4Matrix.expand(w) for w in m.gate_up], [Mxfp4Matrix.expand(w) for w in m.down], m.H, m.I)

    def workspace_bytes(self, T: int, k: int) -> int:
        return int(_abi.load().mxfp4_grouped_moe_workspace(ctypes.byref(self._moe), T, k))

    def hidden_offset(self, T: int, k: int) -> int:
        return int(_abi.load().mxfp4_grouped_moe_hidden_offset(ctypes.byref(self._moe), T, k))


def mxfp4_grouped_moe(m: Mxfp4MoEWeights, x: torch.Tensor, ids: torch.Tensor, wts: torch.Tensor, out=None,
                      workspace=None):
    """The grouped MoE layer of grouped_moe, from resident MXFP4 experts."""
    T, k = ids.shape
    if out is None:
        out = torch.empty((T, m.H), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(m.workspace_bytes(T, k), 1), dtype=torch.uint8, device=x.device)
    _abi.check(_abi.load().mxfp4_grouped_moe(ctypes.byref(m._moe), _ptr(x), T, _ptr(ids), _ptr(wts), k, _ptr(out),
                                             _ptr(workspace), workspace.numel(), _stream_handle()),
               "mxfp4_grouped_moe")
    return out, workspace


def encode_workspace_bytes(rows: int, cols: int, seg_len: int) -> int:
    return int(_abi.load().trellis_encode_workspace(rows, cols, seg_len))


def encode(target: torch.Tensor, D: torch.Tensor, scales: torch.Tensor, seg_len: int = 32, workspace=None):
    """D-weighted Viterbi encoding of fp64 target [rows][cols] under UE8M0 block scales [rows][cols/32]:
    returns (a TrellisMatrix holding the stream and those scales, per-segment minimum costs fp64)."""
    rows, cols = target.shape
    st = torch.empty(rows * (cols // 32) * 2, dtype=torch.int32, device=target.device)
    cost = torch.empty((rows, cols // seg_len), dtype=torch.float64, device=target.device)
    if workspace is None:
        workspace = torch.empty(max(encode_workspace_bytes(rows, cols, seg_len), 1), dtype=torch.uint8,
                                device=target.device)
    _abi.check(_abi.load().trellis_encode(_ptr(target), _ptr(D), _ptr(scales), rows, cols, seg_len, _ptr(st),
                                          _ptr(cost), _ptr(workspace), workspace.numel(), _stream_handle()),
               "trellis_encode")
    return TrellisMatrix(st, scales.reshape(-1), rows, cols, seg_len), cost


def moe_workspace_bytes(m: MoEWeights, T: int, k: int) -> int:
    return m.workspace_bytes(T, k)


def moe_hidden_offset(m: MoEWeights, T: int, k: int) -> int:
    return m.hidden_offset(T, k)


def grouped_moe(m: MoEWeights, x: torch.Tensor, ids: torch.Tensor, wts: torch.Tensor, out=None, workspace=None):
    """out[t] = bf16(sum_j w[t][j] * down_j(bf16(silu(g) * u))) with the stream decoded in-kernel."""
    T, k = ids.shape
    if out is None:
        out = torch.empty((T, m.H), dtype=torch.bfloat16, device=x.device)
    need = m.workspace_bytes(T, k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _abi.check(_abi.load().trellis_grouped_moe(ctypes.byref(m._moe), _ptr(x), T, _ptr(ids), _ptr(wts), k, _ptr(out),
                                               _ptr(workspace), workspace.numel(), _stream_handle()),
               "trellis_grouped_moe")
    return out, workspace


def device_timeouts() -> int:
    """Bounded waits that gave up in the library's kernels since the last query (synchronizes)."""
    return int(_abi.load().tcf4_device_timeouts())
