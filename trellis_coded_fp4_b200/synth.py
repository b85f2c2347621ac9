"""Seeded synthetic inputs for the trellis-coded FP4 path.

This module only draws random inputs; it holds none of the method's arithmetic (no decoding, no
products). Both the CUDA tests/bench and the oracle tests take their inputs from here.

Recipe (the workloads the pages describe are MoE expert weights served from a compressed
trellis stream; no dataset or trained weights are used):

* trellis stream: uniform random bits, [rows][cols/32][2] uint32 (one pair of words per
  32-weight block), i.e. uniform random 2-bit branch symbols;
* block scales: UE8M0 bytes, uniform integers in [lo, hi] (120..126, or 118..126 for the
  hidden-7168 layer), [rows][cols/32] uint8;
* activations: N(0,1) drawn in fp32 and rounded to bf16 (round to nearest even);
* router logits: N(0,1) fp32.

Seeds: ``0x7CF40000 + workload id``; every tensor draws from its own stream,
``np.random.default_rng([seed, tensor_tag])``.
"""
from dataclasses import dataclass

import numpy as np
import torch

SEED_BASE = 0x7CF40000

# tensor tags (second word of the seed sequence), so every tensor has its own random stream
TAG_STREAM, TAG_SCALES, TAG_X, TAG_LOGITS, TAG_GU, TAG_GUS, TAG_DN, TAG_DNS, TAG_MISC = range(9)


def rng(seed: int, tag: int, sub: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed) & 0xFFFFFFFF, int(tag), int(sub)])


def stream(rows: int, cols: int, seed: int, tag: int = TAG_STREAM, sub: int = 0) -> np.ndarray:
    """Uniform random trellis words, [rows][cols/32][2] uint32."""
    assert cols % 32 == 0
    n = rows * (cols // 32) * 2
    raw = rng(seed, tag, sub).bytes(4 * n)
    return np.frombuffer(raw, dtype=np.uint32).reshape(rows, cols // 32, 2).copy()


def scales(rows: int, cols: int, seed: int, lo: int = 120, hi: int = 126, tag: int = TAG_SCALES,
           sub: int = 0) -> np.ndarray:
    """UE8M0 exponent bytes uniform in [lo, hi], [rows][cols/32] uint8."""
    assert cols % 32 == 0 and 0 <= lo <= hi <= 254
    return rng(seed, tag, sub).integers(lo, hi + 1, size=(rows, cols // 32), dtype=np.uint8)


def activations(T: int, K: int, seed: int, sub: int = 0) -> torch.Tensor:
    """bf16 N(0,1) activations [T][K] (CPU tensor)."""
    x = rng(seed, TAG_X, sub).standard_normal((T, K), dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a bf16 tensor."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def logits(T: int, E: int, seed: int, sub: int = 0) -> torch.Tensor:
    """fp32 N(0,1) router logits [T][E] (CPU tensor)."""
    return torch.from_numpy(rng(seed, TAG_LOGITS, sub).standard_normal((T, E), dtype=np.float32))


@dataclass
class MoELayer:
    """All experts of one MoE layer, stored contiguously per kind:
    gate_up [E][2I][H] (gate rows 0..I-1, up rows I..2I-1) and down [E][H][I]."""
    E: int
    H: int
    I: int
    gu_stream: np.ndarray   # [E][2I][H/32][2] uint32
    gu_scales: np.ndarray   # [E][2I][H/32] uint8
    dn_stream: np.ndarray   # [E][H][I/32][2] uint32
    dn_scales: np.ndarray   # [E][H][I/32] uint8


def moe_layer(E: int, H: int, I: int, seed: int, lo: int = 120, hi: int = 126) -> MoELayer:
    assert H % 32 == 0 and I % 32 == 0
    gu = stream(E * 2 * I, H, seed, TAG_GU).reshape(E, 2 * I, H // 32, 2)
    gus = scales(E * 2 * I, H, seed, lo, hi, TAG_GUS).reshape(E, 2 * I, H // 32)
    dn = stream(E * H, I, seed, TAG_DN).reshape(E, H, I // 32, 2)
    dns = scales(E * H, I, seed, lo, hi, TAG_DNS).reshape(E, H, I // 32)
    return MoELayer(E, H, I, gu, gus, dn, dns)
