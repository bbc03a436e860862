"""Packing kernel vs the oracle: codes, scales and zero points bit for bit."""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from w4_gemm_error_b200.inputs import make_layer, to_bf16

pytestmark = pytest.mark.gpu


def _gpu_pack(W: torch.Tensor):
    from w4_gemm_error_b200.spear import W4ECLinear
    lin = W4ECLinear(W.cuda(), None, None, None, 0.0, max_M=1)
    codes, s, z = lin.packed()
    st = lin.status()
    lin.close()
    return codes.cpu().numpy().view(np.uint32), s.cpu().numpy(), z.cpu().numpy(), st


def _check(W: torch.Tensor):
    c_ref, s_ref, z_ref = oracle.pack(W)
    c, s, z, st = _gpu_pack(W)
    assert st == 0
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    assert np.array_equal(z, z_ref), "zero points differ"
    if not np.array_equal(c, c_ref):
        bad = np.argwhere(c != c_ref)[0]
        raise AssertionError(f"codes differ at word {tuple(bad)}: {c[tuple(bad)]:#010x} vs {c_ref[tuple(bad)]:#010x}")


@pytest.mark.parametrize("K,N", [(256, 256), (4096, 4096), (4096, 14336), (14336, 4096), (2048, 512)])
def test_pack_bit_exact_llama_shapes(K, N):
    _check(make_layer(K, N, 0, seed=1).W)


def test_pack_bit_exact_prefill_heavy_rows():
    _check(make_layer(4096, 1024, 0, seed=2, w_row_outlier_frac=0.005).W)


@pytest.mark.parametrize("K,N", [(8, 8), (136, 40), (1000, 24), (264, 136)])
def test_pack_ragged_shapes(K, N):
    rng = np.random.default_rng(K * 31 + N)
    _check(to_bf16(rng.standard_normal((N, K)) * 0.02))


def test_pack_golden_rows_and_edge_rows():
    here = os.path.dirname(os.path.abspath(__file__))
    rows = []
    for line in open(os.path.join(here, "golden", "pack_rows_k16.txt")):
        line = line.split("#")[0].split()
        if line and line[0].startswith("row"):
            rows.append([float(v) for v in line[1:]])
    W = np.array(rows)
    tiny = np.full((1, 16), 2.0 ** -130)           # subnormal amax: no flush to zero
    tiny[0, 3] = -(2.0 ** -129)
    huge = np.full((1, 16), 3.0e38)
    huge[0, 5] = -1.0
    ties = np.array([[0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5, 7.0, -0.5, -1.5, -2.5, -3.5, -4.5, -5.5, -6.5, 0.0]])
    _check(to_bf16(np.concatenate([W, tiny, huge, ties, np.zeros((1, 16))])))


def test_pack_flags_non_finite_weights():
    W = to_bf16(np.ones((16, 64)))
    W[3, 7] = float("nan")
    _, _, _, st = _gpu_pack(W)
    from w4_gemm_error_b200.spear import SPEAR_ERR_DEVICE
    assert st == SPEAR_ERR_DEVICE
