"""GPU parity for the grouped MoE layer with in-kernel trellis decode (two-stage check)."""
import numpy as np
import pytest
import torch

import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import synth

from gpu_common import check_moe

pytestmark = pytest.mark.gpu


def _run(layer, T, k, seed, seg=32, seg_dn=None, ids=None, wts=None):
    W = tc.MoEWeights.from_layer(layer, seg_len=seg, seg_len_down=seg_dn)
    x = synth.activations(T, layer.H, seed=seed).cuda()
    if ids is None:
        ids, wts = tc.moe_route(synth.logits(T, layer.E, seed=seed).cuda(), k)
    out, ws = tc.grouped_moe(W, x, ids, wts)
    torch.cuda.synchronize()
    return W, x, ids, wts, out, ws


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("seg", [32, "full"])
def test_moe_small(T, seg):
    E, H, I, k = 8, 64, 96, 2
    layer = synth.moe_layer(E, H, I, seed=4000 + T)
    seg_gu, seg_dn = (32, 32) if seg == 32 else (H, I)   # "full": one segment per row
    W, x, ids, wts, out, ws = _run(layer, T, k, 4000 + T, seg=seg_gu, seg_dn=seg_dn)
    check_moe(layer, W, x, ids, wts, out, ws, k, seg_gu, seg_dn)


def test_moe_all_tokens_on_the_same_experts():
    # Forced skew: every token routed to the same k experts, so one decode serves all T tokens
    # (more tokens than one pass holds).
    E, H, I, k, T = 6, 128, 64, 3, 11
    layer = synth.moe_layer(E, H, I, seed=4100)
    ids = torch.tensor([[4, 1, 2]] * T, dtype=torch.int32).cuda()
    wts = torch.rand(T, k, generator=torch.Generator().manual_seed(4100)).cuda()
    W, x, ids, wts, out, ws = _run(layer, T, k, 4100, ids=ids, wts=wts)
    check_moe(layer, W, x, ids, wts, out, ws, k, 32)


def test_moe_invalid_expert_ids_contribute_nothing():
    E, H, I, k, T = 5, 64, 64, 2, 3
    layer = synth.moe_layer(E, H, I, seed=4200)
    ids = torch.tensor([[0, -1], [7, 3], [2, 2]], dtype=torch.int32).cuda()
    wts = torch.tensor([[0.5, 0.5], [0.25, 0.75], [0.6, 0.4]], dtype=torch.float32).cuda()
    W, x, ids, wts, out, ws = _run(layer, T, k, 4200, ids=ids, wts=wts)
    check_moe(layer, W, x, ids, wts, out, ws, k, 32)


def test_moe_32_experts_hidden_2880_batch1():
    # The 32-expert, hidden-2880, top-4 layer at batch 1, fully checked.
    E, H, I, k, T = 32, 2880, 2880, 4, 1
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 2)
    W, x, ids, wts, out, ws = _run(layer, T, k, synth.SEED_BASE + 2)
    check_moe(layer, W, x, ids, wts, out, ws, k, 32)


@pytest.mark.parametrize("T", [2, 4, 8, 16, 32])
def test_moe_32_experts_batch_sweep_sampled(T):
    E, H, I, k = 32, 2880, 2880, 4
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 3)
    W, x, ids, wts, out, ws = _run(layer, T, k, synth.SEED_BASE + 3 + T)
    r = np.random.default_rng(T)
    check_moe(layer, W, x, ids, wts, out, ws, k, 32, rows_h=r.choice(I, 48, replace=False),
              rows_out=r.choice(H, 48, replace=False))


@pytest.fixture(scope="module")
def layer_7168():
    # 256 experts, hidden 7168, intermediate 2048 (11.3 G weights, 3.17 GB resident), built once
    E, H, I = 256, 7168, 2048
    layer = synth.moe_layer(E, H, I, seed=synth.SEED_BASE + 4, lo=118, hi=126)
    return layer, tc.MoEWeights.from_layer(layer, seg_len=32)


@pytest.mark.parametrize("T", [1, 8, 32])
def test_moe_256_experts_hidden_7168_sampled(layer_7168, T):
    layer, W = layer_7168
    k = 8
    x = synth.activations(T, layer.H, seed=synth.SEED_BASE + 4 + T).cuda()
    ids, wts = tc.moe_route(synth.logits(T, layer.E, seed=synth.SEED_BASE + 4 + T).cuda(), k)
    out, ws = tc.grouped_moe(W, x, ids, wts)
    torch.cuda.synchronize()
    r = np.random.default_rng(100 + T)
    check_moe(layer, W, x, ids, wts, out, ws, k, 32, rows_h=r.choice(layer.I, 24, replace=False),
              rows_out=r.choice(layer.H, 24, replace=False))


def test_moe_tensor_core_path_many_tokens_per_expert():
    # K = 1024 takes the tensor-core path; 20 tokens on each of two experts split into groups of 16
    # and 4 columns pairs of the MMA.
    E, H, I, k, T = 8, 1024, 1024, 2, 20
    layer = synth.moe_layer(E, H, I, seed=4300)
    ids = torch.tensor([[1, 5]] * T, dtype=torch.int32).cuda()
    wts = torch.rand(T, k, generator=torch.Generator().manual_seed(4300)).cuda()
    W, x, ids, wts, out, ws = _run(layer, T, k, 4300, ids=ids, wts=wts)
    r = np.random.default_rng(4300)
    check_moe(layer, W, x, ids, wts, out, ws, k, 32, rows_h=r.choice(I, 64, replace=False),
              rows_out=r.choice(H, 64, replace=False))


def test_no_bounded_wait_gave_up():
    # Every bulk-copy wait in the kernels above completed within its iteration limit.
    assert tc.device_timeouts() == 0
