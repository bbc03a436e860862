"""Shared helpers of the GPU parity tests: problem setup, the tolerance check.

Tolerance (floating point outputs, written here once):
    elementwise |y - y_ref| <= 1e-2 + 1e-2 * |y_ref|   and
    ||y - y_ref||_F / ||y_ref||_F <= 5e-3,
with y_ref the fp64 oracle.  Codes, scales and zero points are compared bit
for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from w4_gemm_error_b200.inputs import make_layer, make_x

ATOL = 1e-2
RTOL = 1e-2
FROB = 5e-3


def assert_close(y: torch.Tensor, ref: np.ndarray, what: str = "y"):
    y = y.detach().float().cpu().double().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    err = np.abs(y - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; first at {tuple(i)}: "
                             f"got {y[tuple(i)]!r}, want {ref[tuple(i)]!r}")
    nref = np.linalg.norm(ref)
    if nref > 0:
        frob = np.linalg.norm(y - ref) / nref
        assert frob <= FROB, f"{what}: relative Frobenius error {frob:.3e} > {FROB}"


class Problem:
    """A seeded layer + activations, its GPU handle and the oracle's view of it."""

    def __init__(self, M, K, N, r, seed=0, max_M=None, device="cuda", **layer_kw):
        from w4_gemm_error_b200.spear import W4ECLinear
        x_frac = layer_kw.pop("x_outlier_frac", 0.01)
        self.layer = make_layer(K, N, r, seed=seed, x_outlier_frac=x_frac, **layer_kw)
        self.x = make_x(M, K, seed=seed, x_outlier_frac=x_frac)
        self.M, self.K, self.N, self.r = M, K, N, r
        L = self.layer
        dev = torch.device(device)
        self.xd = self.x.to(dev)
        self.lin = W4ECLinear(L.W.to(dev), L.A.to(dev) if r else None, L.B.to(dev) if r else None,
                              L.wg.to(dev) if r else None, L.b_g, max_M=max_M or max(M, 1))
        self._packed = None

    def oracle_packed(self):
        if self._packed is None:
            self._packed = oracle.pack(self.layer.W)
        return self._packed

    def oracle_y(self, ec_on=True, want_corr=False):
        codes, s, z = self.oracle_packed()
        L = self.layer
        return oracle.forward(self.x, codes, s, z, L.A, L.B, L.wg, L.b_g, ec_on=ec_on, want_corr=want_corr)

    def oracle_sampled(self, t_idx, n_idx, ec_on=True):
        codes, s, z = self.oracle_packed()
        L = self.layer
        return oracle.forward_sampled(self.x, codes, s, z, L.A, L.B, L.wg, L.b_g, t_idx, n_idx, ec_on=ec_on)

    def close(self):
        self.lin.close()


def tc_token_tile(M: int) -> int:
    """Token width of the tcgen05 kernel's output tile: the narrowest of 32,
    64, 128 and 256 that holds M tokens (the tile is 128 weight rows high)."""
    return 32 if M <= 32 else (64 if M <= 64 else (128 if M <= 128 else 256))


def per_tile_samples(M: int, N: int, tile_t: int, tile_n: int = 128, per_tile: int = 4, seed: int = 0):
    """Output indices (t, n) that hit every tile_t x tile_n output tile at
    least ``per_tile`` times: the tile's first and last output (clipped to
    the ragged edge of y) and per_tile - 2 seeded interior ones, so that a
    tile no launch wrote, or one written with another tile's accumulator,
    cannot hide between random samples."""
    rng = np.random.default_rng(seed)
    ts, ns = [], []
    for t0 in range(0, M, tile_t):
        t1 = min(M, t0 + tile_t)
        for n0 in range(0, N, tile_n):
            n1 = min(N, n0 + tile_n)
            ts += [t0, t1 - 1]
            ns += [n0, n1 - 1]
            ts += list(rng.integers(t0, t1, per_tile - 2))
            ns += list(rng.integers(n0, n1, per_tile - 2))
    return np.asarray(ts, dtype=np.int64), np.asarray(ns, dtype=np.int64)
