"""The allocation-free gate entry point against the handle-based one.

spear_w4ec_gate_noalloc serves callers that may not call cudaMalloc (code
under CUDA graph capture, fixed-budget serving loops, hosts whose memory pool
owns every allocation): it takes the caller's x and w_g and keeps its
scratch in a static device array.  Its gate must match spear_w4ec_get_gate's
within the gate tolerance of the other tests (1e-5 absolute), on two calls
in a row (the scratch keeps the previous call's contents).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from w4_gemm_error_b200.inputs import make_layer, make_x

pytestmark = pytest.mark.gpu

GATE_TOL = 1e-5


def test_noalloc_gate_matches_handle_gate_twice():
    from w4_gemm_error_b200 import spear
    K, N, r = 4096, 256, 32
    lay = make_layer(K, N, r, seed=21, gate_open_frac=0.3)
    lin = spear.W4ECLinear(lay.W.cuda(), lay.A.cuda(), lay.B.cuda(), lay.wg.cuda(), lay.b_g, max_M=4096)
    wg = lay.wg.cuda()
    lib = spear.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call, M in enumerate((37, 4096)):       # two calls in a row, different sizes
        x = make_x(M, K, seed=100 + call).cuda()
        g_ref = lin.gate(x)
        g = torch.full((M,), float("nan"), device="cuda")
        rc = lib.spear_w4ec_gate_noalloc(x.data_ptr(), M, K, wg.data_ptr(), float(lay.b_g), g.data_ptr(), stream)
        assert rc == spear.SPEAR_OK, spear.strerror(rc)
        torch.cuda.synchronize()
        diff = (g.double() - g_ref.double()).abs().max().item()
        assert np.isfinite(diff) and diff <= GATE_TOL, (call, diff)
    lin.close()


def test_noalloc_gate_rejects_sizes_beyond_its_scratch():
    from w4_gemm_error_b200 import spear
    lib = spear.lib()
    x = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    wg = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert lib.spear_w4ec_gate_noalloc(x.data_ptr(), 4097, 64, wg.data_ptr(), 0.0, g.data_ptr(), s) \
        == spear.SPEAR_ERR_INVALID
    assert lib.spear_w4ec_gate_noalloc(x.data_ptr(), 8, 60, wg.data_ptr(), 0.0, g.data_ptr(), s) \
        == spear.SPEAR_ERR_INVALID
    assert lib.spear_w4ec_gate_noalloc(x.data_ptr(), 0, 64, wg.data_ptr(), 0.0, g.data_ptr(), s) == spear.SPEAR_OK
