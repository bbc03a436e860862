"""Asymmetric (min-max, stored zero point) packing and the import of codes
quantised elsewhere, against the oracle.

SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
Efficient Low-Bit LLM Serving", Abstract: the Error Compensators sit on top
of existing 4-bit per-channel quantizers.  spear_w4ec_pack_asym must give the
oracle's codes, scales and zero points bit for bit; spear_w4ec_import must
keep any codes / scales / zero points it is given bit for bit; and the
forward pass must match the oracle on layers with zero points other than 8,
on every kernel family (decode and tcgen05, EC fused and split, EC off).
"""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close, per_tile_samples, tc_token_tile
from w4_gemm_error_b200.inputs import make_layer, make_x, to_bf16

pytestmark = pytest.mark.gpu

FUSED, SPLIT, DECODE, TC, EC_OFF = 2, 4, 8, 16, 1


def _gpu_pack_asym(W: torch.Tensor):
    from w4_gemm_error_b200.spear import W4ECLinear
    lin = W4ECLinear(W.cuda(), None, None, None, 0.0, max_M=1, quant="asym")
    codes, s, z = lin.packed()
    st = lin.status()
    lin.close()
    return codes.cpu().numpy().view(np.uint32), s.cpu().numpy(), z.cpu().numpy(), st


def _check(W: torch.Tensor):
    c_ref, s_ref, z_ref = oracle.pack_asym(W)
    c, s, z, st = _gpu_pack_asym(W)
    assert st == 0
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32)), "scales differ"
    assert np.array_equal(z, z_ref), "zero points differ"
    if not np.array_equal(c, c_ref):
        bad = np.argwhere(c != c_ref)[0]
        raise AssertionError(f"codes differ at word {tuple(bad)}: {c[tuple(bad)]:#010x} vs {c_ref[tuple(bad)]:#010x}")
    return z_ref


@pytest.mark.parametrize("K,N", [(256, 256), (4096, 4096), (4096, 14336), (14336, 4096)])
def test_pack_asym_bit_exact_llama_shapes(K, N):
    # a per-row offset makes the rows' ranges lopsided, so zero points spread over 0..15
    lay = make_layer(K, N, 0, seed=3)
    rng = np.random.default_rng(K + N)
    W = to_bf16(lay.W.double().numpy() + rng.standard_normal((N, 1)) * 0.03)
    z = _check(W)
    assert len(np.unique(z)) >= 8


@pytest.mark.parametrize("K,N", [(8, 8), (136, 40), (1000, 24), (264, 136)])
def test_pack_asym_ragged_shapes(K, N):
    rng = np.random.default_rng(K * 37 + N)
    _check(to_bf16(rng.standard_normal((N, K)) * 0.02 + rng.standard_normal((N, 1)) * 0.02))


def test_pack_asym_golden_and_edge_rows():
    here = os.path.dirname(os.path.abspath(__file__))
    rows = []
    for line in open(os.path.join(here, "golden", "pack_asym_rows_k16.txt")):
        line = line.split("#")[0].split()
        if line and line[0].startswith("row"):
            rows.append([float(v) for v in line[1:]])
    W = np.array(rows)
    tiny = np.full((1, 16), 2.0 ** -130)            # subnormal range: no flush to zero
    tiny[0, 3] = -(2.0 ** -129)
    rng = np.random.default_rng(1)
    pos = np.abs(rng.standard_normal((2, 16)))       # all-positive and all-negative rows
    neg = -np.abs(rng.standard_normal((2, 16)))
    one = np.zeros((1, 16))
    one[0, 9] = -3.0                                  # a single nonzero weight
    const = np.full((1, 16), 0.75)                    # a constant row
    huge = np.full((1, 16), 3.0e38)                    # range near the top of fp32
    huge[0, 5] = -1.0
    ztie = np.linspace(-0.3125, 1.5625, 16)[None, :]  # -lo / s = 2.5: the zero point ties to 2
    ztie = np.round(ztie * 64) / 64
    ztie[0, 0], ztie[0, -1] = -0.3125, 1.5625
    alt = np.tile([0.5, -0.5], 8)[None, :]
    rows = np.concatenate([W, tiny, pos, neg, one, const, huge, ztie, alt, np.zeros((1, 16))])
    assert rows.shape[0] % 8 == 0                     # N must be a multiple of 8
    _check(to_bf16(rows))


def test_import_keeps_codes_scales_and_zero_points():
    """Random codes (every nibble value), scales and zero points 0..15, on a
    ragged shape: get_packed returns them bit for bit, and the forward pass
    matches the oracle on the same arrays."""
    from w4_gemm_error_b200.spear import W4ECLinear
    rng = np.random.default_rng(7)
    M, K, N, r = 9, 1032, 264, 20
    lay = make_layer(K, N, r, seed=8)
    codes = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = (rng.random(N).astype(np.float32) * np.float32(0.01) + np.float32(1e-3)).astype(np.float32)
    s[5] = 0.0
    z = rng.integers(0, 16, size=N).astype(np.uint8)
    dev = torch.device("cuda")
    packed = (torch.from_numpy(codes.view(np.int32)).to(dev), torch.from_numpy(s).to(dev),
              torch.from_numpy(z).to(dev))
    lin = W4ECLinear(None, lay.A.cuda(), lay.B.cuda(), lay.wg.cuda(), lay.b_g, max_M=64, packed=packed)
    c2, s2, z2 = lin.packed()
    assert lin.status() == 0
    assert np.array_equal(c2.cpu().numpy().view(np.uint32), codes)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s.view(np.uint32))
    assert np.array_equal(z2.cpu().numpy(), z)
    for Mx in (M, 40):
        x = make_x(Mx, K, seed=9)
        ref = oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g)
        flag_sets = (0, DECODE | FUSED, DECODE | SPLIT, TC | FUSED, TC | SPLIT) if Mx <= 32 else \
            (0, TC | FUSED, TC | SPLIT)
        for flags in flag_sets:
            y = lin(x.cuda(), flags)
            torch.cuda.synchronize()
            assert lin.status() == 0
            assert_close(y, ref, f"M={Mx} flags={flags}")
    lin.close()


def test_import_flags_bad_zero_points_and_scales():
    from w4_gemm_error_b200.spear import W4ECLinear, SPEAR_ERR_DEVICE
    dev = torch.device("cuda")
    codes = torch.zeros((16, 8), dtype=torch.int32, device=dev)
    for s_bad, z_bad in ((0.01, 16), (float("inf"), 3)):
        s = torch.full((16,), 0.01, device=dev)
        z = torch.full((16,), 8, dtype=torch.uint8, device=dev)
        s[3] = s_bad
        z[3] = z_bad
        lin = W4ECLinear(None, None, None, None, 0.0, max_M=1, packed=(codes, s, z))
        assert lin.status() == SPEAR_ERR_DEVICE
        lin.close()


@pytest.mark.parametrize("M,K,N,r", [(1, 4096, 4096, 32), (16, 4096, 4096, 32), (5, 1032, 264, 20),
                                     (16, 14336, 4096, 64), (37, 2048, 512, 32), (300, 1024, 1024, 32)])
def test_forward_asym_layers_match_oracle(M, K, N, r):
    """Zero points other than 8 through every kernel family."""
    from w4_gemm_error_b200.spear import W4ECLinear
    lay = make_layer(K, N, r, seed=M + K)
    rng = np.random.default_rng(M + N)
    W = to_bf16(lay.W.double().numpy() + rng.standard_normal((N, 1)) * 0.03)
    x = make_x(M, K, seed=M)
    codes, s, z = oracle.pack_asym(W)
    assert np.count_nonzero(z != 8) > N // 2
    lin = W4ECLinear(W.cuda(), lay.A.cuda(), lay.B.cuda(), lay.wg.cuda(), lay.b_g, max_M=M, quant="asym")
    ref = oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g)
    ref_off = oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g, ec_on=False)
    paths = [0, TC | FUSED, TC | SPLIT] + ([DECODE | FUSED, DECODE | SPLIT] if M <= 32 else [])
    for flags in paths:
        y = lin(x.cuda(), flags)
        torch.cuda.synchronize()
        assert lin.status() == 0
        assert_close(y, ref, f"flags={flags}")
    y = lin(x.cuda(), EC_OFF)
    torch.cuda.synchronize()
    assert_close(y, ref_off, "EC off")
    lin.close()
