"""The allocation-free gate entry point against the fp64 oracle and the
handle-based one.

spear_w4ec_gate_noalloc serves callers that may not call cudaMalloc (code
under CUDA graph capture, fixed-budget serving loops, hosts whose memory pool
owns every allocation): it takes the caller's x and w_g and keeps its
scratch in a static device array.  Its gate must match the oracle's and
spear_w4ec_get_gate's within the gate tolerance of the other tests (1e-5
absolute), on several calls in a row (the scratch keeps the previous call's
contents): split-K calls of 37, 4095 (a ragged last tile) and 4096 tokens,
and a K = 64 call whose single split writes the gate directly.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from w4_gemm_error_b200.inputs import make_layer, make_x

pytestmark = pytest.mark.gpu

GATE_TOL = 1e-5


def test_noalloc_gate_matches_oracle_and_handle_gate_on_calls_in_a_row():
    import oracle
    from w4_gemm_error_b200 import spear
    lib = spear.lib()
    stream = torch.cuda.current_stream().cuda_stream
    lins = {}
    # calls in a row on the same static scratch, different sizes and split counts
    for call, (M, K) in enumerate(((37, 4096), (4095, 4096), (5, 64), (4096, 4096))):
        if K not in lins:
            lay = make_layer(K, 256, 32, seed=21 + K, gate_open_frac=0.3)
            lins[K] = (lay, spear.W4ECLinear(lay.W.cuda(), lay.A.cuda(), lay.B.cuda(), lay.wg.cuda(), lay.b_g,
                                             max_M=4096), lay.wg.cuda())
        lay, lin, wg = lins[K]
        x_host = make_x(M, K, seed=100 + call)
        x = x_host.cuda()
        g = torch.full((M,), float("nan"), device="cuda")
        rc = lib.spear_w4ec_gate_noalloc(x.data_ptr(), M, K, wg.data_ptr(), float(lay.b_g), g.data_ptr(), stream)
        assert rc == spear.SPEAR_OK, spear.strerror(rc)
        torch.cuda.synchronize()
        got = g.double().cpu().numpy()
        assert np.all(np.isfinite(got)), call
        ref = oracle.gate(x_host, lay.wg, lay.b_g)
        assert np.max(np.abs(got - ref)) <= GATE_TOL, (call, M, K, np.max(np.abs(got - ref)))
        g_handle = lin.gate(x).double().cpu().numpy()
        assert np.max(np.abs(got - g_handle)) <= GATE_TOL, (call, M, K)
    for _, lin, _ in lins.values():
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
