"""trellis_gemv_noalloc against trellis_gemv (and the oracle), two calls in a row.

This file is collected last so that it runs both after every other GPU test and, when run alone,
in a fresh process (then its first call is the one that does the per-device setup).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import trellis_coded_fp4_b200 as tc
from trellis_coded_fp4_b200 import _abi, synth

from gpu_common import assert_products_close, bf16_to_f64, xnorms

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,cols,T", [(1000, 2880, 1), (300, 7168, 5), (129, 1024, 16), (130, 16384, 32)])
def test_noalloc_matches_workspace_entry_point(rows, cols, T):
    st = synth.stream(rows, cols, seed=7000 + T)
    sc = synth.scales(rows, cols, seed=7000 + T)
    W = tc.TrellisMatrix.from_numpy(st, sc, rows, cols, 32)
    L = _abi.load()
    assert L.trellis_gemv_workspace(W.abi(), T) > 0          # the tensor-core path, which uses scratch
    y_ref = tc.gemv(W, synth.activations(T, cols, seed=7100 + T).cuda())
    exact, wn = oracle.gemv(st, sc, rows, cols, 32, synth.bf16_bits(synth.activations(T, cols, seed=7100 + T)))
    for call in range(2):                                    # the second call reuses the scratch
        x = synth.activations(T, cols, seed=7100 + T).cuda()
        y = torch.full((T, rows), float("nan"), dtype=torch.bfloat16, device="cuda")
        st_code = L.trellis_gemv_noalloc(W.abi(), ctypes.c_void_p(x.data_ptr()), T, ctypes.c_void_p(y.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        torch.cuda.synchronize()
        assert st_code == 0, _abi.STATUS_NAMES.get(st_code, st_code)
        assert_products_close(y, exact, wn, xnorms(synth.bf16_bits(x.cpu())), f"noalloc call {call}", cols=cols)
        assert (bf16_to_f64(y) == bf16_to_f64(y_ref)).all()  # same kernels, same scratch contents
    assert L.tcf4_device_timeouts() == 0
