"""Pins of the fp64 CPU oracle against facts other than itself (CPU only).

Each pin checks the oracle against a hand-derived worked example, exact
rational arithmetic, a closed form, or a library routine in a special case
(NumPy fp64 matmul when the gate is fully closed or fully open).  The last
test plants plausible mistakes in copies of the oracle and checks that every
mutant fails at least one pin, so a wrong oracle cannot pass unnoticed.

The layer (SPEAR, "A System for Post-Quantization Error-Adaptive Recovery
Enabling Efficient Low-Bit LLM Serving", Abstract): a 4-bit per-channel
linear, corrected by a lightweight Error Compensator gated per token.
"""
from __future__ import annotations

import math
import os
import re
import subprocess
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from w4_gemm_error_b200.inputs import bf16_bits, make_layer, make_x, to_bf16

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _bits(vals) -> np.ndarray:
    return bf16_bits(to_bf16(np.asarray(vals, dtype=np.float64)))


def _exact_bf16(vals) -> np.ndarray:
    """Assert the values are bf16-exact and return their bit patterns."""
    b = _bits(vals)
    back = torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    assert np.array_equal(back, np.asarray(vals, dtype=np.float64)), "fixture value not bf16-exact"
    return b


def _quantizable_W(rng, N, K, emin=-9, emax=-1):
    """W[n,k] = 2^e_n * (q - 8) with a |q-8| = 7 entry in every row, so the
    per-channel RTN quantiser reproduces W exactly (s = 2^e_n)."""
    q = rng.integers(1, 16, size=(N, K))
    q[np.arange(N), rng.integers(0, K, size=N)] = rng.choice([1, 15], size=N)
    e = rng.integers(emin, emax + 1, size=N)
    W = (q - 8).astype(np.float64) * np.exp2(e)[:, None]
    return W, q, e


def _dyadic(rng, shape, lo=-8, hi=8, denom=4):
    return rng.integers(lo, hi + 1, size=shape).astype(np.float64) / denom


# --------------------------------------------------------------------------- pins

def pin_pack_golden(lib=None):
    blocks = {}
    with open(os.path.join(GOLDEN, "pack_rows_k16.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            blocks[key] = vals
    rows = sorted(int(k[3:]) for k in blocks if k.startswith("row"))
    W = np.array([[float(v) for v in blocks[f"row{i}"]] for i in rows])
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    for i in rows:
        assert s[i].view(np.uint32) == int(blocks[f"s{i}"][0], 16), f"scale of row {i}"
        want_words = [int(w, 16) for w in blocks[f"words{i}"]]
        assert list(codes[i]) == want_words, f"packed words of row {i}"
        got_codes = [(int(codes[i][k // 8]) >> (4 * (k % 8))) & 0xF for k in range(16)]
        assert got_codes == [int(c) for c in blocks[f"codes{i}"]], f"codes of row {i}"
        assert z[i] == 8


def pin_requant_identity(lib=None):
    rng = np.random.default_rng(11)
    W, q, e = _quantizable_W(rng, 40, 64)
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    got = np.stack([(codes[:, k // 8] >> (4 * (k % 8))) & 0xF for k in range(64)], axis=1)
    assert np.array_equal(got, q)
    assert np.array_equal(s.astype(np.float64), np.exp2(e))
    assert np.all(z == 8)


def pin_pack_properties(lib=None):
    rng = np.random.default_rng(5)
    W = to_bf16(rng.standard_normal((64, 128)) * 0.02)
    codes, s, z = oracle.pack(W, lib=lib)
    Wd = W.double().numpy()
    amax = np.abs(Wd).max(axis=1)
    # IEEE fp32 quotient computed natively by NumPy, a route independent of the oracle's
    assert np.array_equal(s, np.float32(amax.astype(np.float32)) / np.float32(7.0))
    q = np.stack([(codes[:, k // 8] >> (4 * (k % 8))) & 0xF for k in range(128)], axis=1).astype(np.int64)
    assert q.min() >= 1 and q.max() <= 15
    w_hat = s.astype(np.float64)[:, None] * (q - 8)
    # round-to-nearest error bound (1 ulp of the fp32 quotient allowed)
    assert np.all(np.abs(Wd - w_hat) <= s.astype(np.float64)[:, None] * (0.5 + 2.0 ** -20))
    # the amax entry of every row maps to +-7
    arg = np.abs(Wd).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(64), arg] - 8) == 7)


def _read_golden_rows(name):
    blocks = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            blocks[key] = vals
    return blocks


def pin_pack_asym_golden(lib=None):
    blocks = _read_golden_rows("pack_asym_rows_k16.txt")
    names = sorted(k[3:] for k in blocks if k.startswith("row"))
    W = np.array([[float(v) for v in blocks[f"row{n}"]] for n in names])
    codes, s, z = oracle.pack_asym(_exact_bf16(W), lib=lib)
    for i, n in enumerate(names):
        assert s[i].view(np.uint32) == int(blocks[f"s{n}"][0], 16), f"scale of row {n}"
        assert int(z[i]) == int(blocks[f"z{n}"][0]), f"zero point of row {n}"
        assert list(codes[i]) == [int(w, 16) for w in blocks[f"words{n}"]], f"packed words of row {n}"
        got = [(int(codes[i][k // 8]) >> (4 * (k % 8))) & 0xF for k in range(16)]
        assert got == [int(c) for c in blocks[f"codes{n}"]], f"codes of row {n}"


def pin_asym_requant_identity(lib=None):
    """W = 2^e (q - z) with a code 0 and a code 15 in every row: the range is
    exactly 15 * 2^e, so the min-max quantiser gives back s = 2^e, z and q
    (zero points 0 and 15 included)."""
    rng = np.random.default_rng(12)
    N, K = 48, 64
    q = rng.integers(0, 16, size=(N, K))
    cols = np.stack([rng.permutation(K)[:2] for _ in range(N)])
    q[np.arange(N), cols[:, 0]] = 0
    q[np.arange(N), cols[:, 1]] = 15
    zp = rng.integers(0, 16, size=N)
    zp[:2] = (0, 15)
    e = rng.integers(-10, -1, size=N)
    W = (q - zp[:, None]).astype(np.float64) * np.exp2(e)[:, None]
    codes, s, z = oracle.pack_asym(_exact_bf16(W), lib=lib)
    got = np.stack([(codes[:, k // 8] >> (4 * (k % 8))) & 0xF for k in range(K)], axis=1)
    assert np.array_equal(got, q)
    assert np.array_equal(z.astype(np.int64), zp)
    assert np.array_equal(s.astype(np.float64), np.exp2(e))


def pin_asym_properties(lib=None):
    """Random rows: the range is the min-max one with 0 kept (scale from an
    IEEE fp32 route of NumPy's own), the zero point maps 0 to a code, and
    every code is a nearest grid point (within half a step, one ulp of the
    fp32 quotient allowed) unless the grid's end clips it (within a step)."""
    rng = np.random.default_rng(6)
    W = to_bf16(rng.standard_normal((64, 128)) * 0.02 + rng.standard_normal((64, 1)) * 0.01)
    codes, s, z = oracle.pack_asym(W, lib=lib)
    Wd = W.double().numpy()
    lo = np.minimum(Wd.min(axis=1), 0.0).astype(np.float32)
    hi = np.maximum(Wd.max(axis=1), 0.0).astype(np.float32)
    assert np.array_equal(s, (hi - lo) / np.float32(15.0))
    q = np.stack([(codes[:, k // 8] >> (4 * (k % 8))) & 0xF for k in range(128)], axis=1).astype(np.int64)
    zf = z.astype(np.float64)[:, None]
    sf = s.astype(np.float64)[:, None]
    assert np.all(np.abs(-lo.astype(np.float64) / s - z) <= 0.5 + 2.0 ** -18)
    w_hat = sf * (q - zf)
    inner = (q > 0) & (q < 15)
    err = np.abs(Wd - w_hat)
    assert np.all(err[inner] <= (sf * (0.5 + 2.0 ** -20) + 0 * Wd)[inner])
    assert np.all(err <= sf * (1.0 + 2.0 ** -20))
    # both ends of every row are used (the range is the row's own)
    assert np.all(q.min(axis=1) <= 1) and np.all(q.max(axis=1) >= 14)


def pin_forward_golden(lib=None):
    vals = {}
    with open(os.path.join(GOLDEN, "forward_2x8x2_r1.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *v = line.split()
            vals.setdefault(key, []).append([float(t) for t in v])
    x = _exact_bf16(vals["x"])
    W = _exact_bf16(vals["W"])
    A = _exact_bf16(np.array(vals["A"]).T)        # [K, 1]
    B = _exact_bf16(vals["B"])                    # [1, N]
    wg = _exact_bf16(vals["wg"][0])
    b_g = vals["b_g"][0][0]
    codes, s, z = oracle.pack(W, lib=lib)
    y, g, _ = oracle.forward(x, codes, s, z, A, B, wg, b_g, want_corr=True, lib=lib)
    assert np.allclose(g, vals["g"][0], rtol=0, atol=1e-15)
    assert np.allclose(y, np.array(vals["y"]), rtol=1e-15, atol=1e-15)


def pin_bruteforce_exact(lib=None):
    """4 tokens x 8 in x 8 out, rank 2: exact rational sums, gate exactly 1/2."""
    rng = np.random.default_rng(3)
    M, K, N, r = 4, 8, 8, 2
    W, _, _ = _quantizable_W(rng, N, K, -3, 0)
    x = _dyadic(rng, (M, K))
    A = _dyadic(rng, (K, r), -4, 4, 8)
    B = _dyadic(rng, (r, N), -4, 4, 8)
    wg = np.zeros(K)
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    y = oracle.forward(_exact_bf16(x), codes, s, z, _exact_bf16(A), _exact_bf16(B), _exact_bf16(wg), 0.0,
                       lib=lib)
    Fx = [[Fraction(v) for v in row] for row in x]
    FW = [[Fraction(v) for v in row] for row in W]
    FA = [[Fraction(v) for v in row] for row in A]
    FB = [[Fraction(v) for v in row] for row in B]
    half = Fraction(1, 2)
    for t in range(M):
        u = [sum((Fx[t][k] * FA[k][j] for k in range(K)), Fraction(0)) for j in range(r)]
        for n in range(N):
            main = sum((Fx[t][k] * FW[n][k] for k in range(K)), Fraction(0))
            corr = half * sum((u[j] * FB[j][n] for j in range(r)), Fraction(0))
            assert abs(y[t, n] - float(main + corr)) <= 1e-12 * (1 + abs(float(main + corr))), (t, n)


def pin_gate_closed_forms(lib=None):
    """sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4, sigmoid(0) = 1/2."""
    K = 16
    x = np.zeros((4, K))
    x[0, 0] = 2.0          # x.w_g = 1
    x[1, 0] = -2.0         # x.w_g = -1
    x[2, 1] = 3.0          # orthogonal to w_g
    wg = np.zeros(K)
    wg[0] = 0.5
    xb, wb = _exact_bf16(x), _exact_bf16(wg)
    g = oracle.gate(xb, wb, math.log(3.0) - 1.0, lib=lib)
    assert abs(g[0] - 0.75) < 1e-15
    assert abs(g[2] - 1.0 / (1.0 + math.e / 3.0)) < 1e-15   # logit ln3 - 1
    g = oracle.gate(xb, wb, 0.0, lib=lib)
    assert abs(g[0] + g[1] - 1.0) < 1e-15 and g[2] == 0.5 and g[3] == 0.5
    g = oracle.gate(xb, wb, -math.log(3.0) + 1.0, lib=lib)
    assert abs(g[1] - 0.25) < 1e-15
    # the gate the forward pass uses is the same one
    codes, s, z = oracle.pack(_exact_bf16(np.ones((8, K))), lib=lib)
    _, gf, _ = oracle.forward(xb, codes, s, z, _exact_bf16(np.zeros((K, 1))), _exact_bf16(np.zeros((1, 8))),
                              wb, math.log(3.0) - 1.0, want_corr=True, lib=lib)
    assert abs(gf[0] - 0.75) < 1e-15


def _numpy_case(rng, M=5, K=24, N=16, r=3):
    W, _, _ = _quantizable_W(rng, N, K)
    x = rng.standard_normal((M, K))
    A = rng.standard_normal((K, r)) * 0.5
    B = rng.standard_normal((r, N)) * 0.5
    wg = rng.standard_normal(K) * 0.2
    xb, Ab, Bb, wb = (to_bf16(v) for v in (x, A, B, wg))
    return W, xb, Ab, Bb, wb


def pin_gate_closed_matches_matmul(lib=None):
    """g == 0 exactly (b_g = -1e4): y is the plain W4 GEMM, x @ W^T."""
    W, xb, Ab, Bb, wb = _numpy_case(np.random.default_rng(21))
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    y = oracle.forward(xb, codes, s, z, Ab, Bb, wb, -1e4, lib=lib)
    ref = xb.double().numpy() @ W.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def pin_gate_open_matches_static_lowrank(lib=None):
    """g == 1 exactly (b_g = +1e4): y = x @ (W^T + A @ B), a static low-rank correction."""
    W, xb, Ab, Bb, wb = _numpy_case(np.random.default_rng(22))
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    y = oracle.forward(xb, codes, s, z, Ab, Bb, wb, 1e4, lib=lib)
    ref = xb.double().numpy() @ (W.T + Ab.double().numpy() @ Bb.double().numpy())
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def pin_rank1_closed_form(lib=None):
    """x = 1, constant rows c_n = +-7*2^e_n, A = alpha, B = beta, gate 1/2:
    y[t,n] = K*c_n + (1/2)*r*alpha*K*beta."""
    M, K, N, r = 3, 40, 6, 5
    e = np.array([-4, -2, 0, -6, -1, -3])
    sign = np.array([1, -1, 1, 1, -1, -1])
    c = sign * 7.0 * np.exp2(e)
    W = np.repeat(c[:, None], K, axis=1)
    alpha, beta = 0.25, -0.75
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    y = oracle.forward(_exact_bf16(np.ones((M, K))), codes, s, z, _exact_bf16(np.full((K, r), alpha)),
                       _exact_bf16(np.full((r, N), beta)), _exact_bf16(np.zeros(K)), 0.0, lib=lib)
    want = K * c + 0.5 * r * alpha * K * beta
    assert np.allclose(y, np.broadcast_to(want, (M, N)), rtol=1e-14, atol=0)


def pin_ec_off_identities(lib=None):
    """EC off == B = 0 == rank 0 (the plain W4 GEMM)."""
    W, xb, Ab, Bb, wb = _numpy_case(np.random.default_rng(23))
    codes, s, z = oracle.pack(_exact_bf16(W), lib=lib)
    y_off = oracle.forward(xb, codes, s, z, Ab, Bb, wb, 0.3, ec_on=False, lib=lib)
    y_b0 = oracle.forward(xb, codes, s, z, Ab, to_bf16(np.zeros(tuple(Bb.shape))), wb, 0.3, lib=lib)
    K, N = xb.shape[1], W.shape[0]
    y_r0 = oracle.forward(xb, codes, s, z, to_bf16(np.zeros((K, 0))), to_bf16(np.zeros((0, N))), wb, 0.3,
                          lib=lib)
    y_on = oracle.forward(xb, codes, s, z, Ab, Bb, wb, 0.3, lib=lib)
    assert np.array_equal(y_off, y_b0) and np.array_equal(y_off, y_r0)
    assert not np.allclose(y_on, y_off)


PINS = [pin_pack_golden, pin_requant_identity, pin_pack_properties, pin_pack_asym_golden,
        pin_asym_requant_identity, pin_asym_properties, pin_forward_golden,
        pin_bruteforce_exact, pin_gate_closed_forms, pin_gate_closed_matches_matmul,
        pin_gate_open_matches_static_lowrank, pin_rank1_closed_form, pin_ec_off_identities]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin()


def test_sampled_equals_full():
    lay = make_layer(64, 48, 8, seed=4)
    x = make_x(7, 64, seed=4)
    codes, s, z = oracle.pack(lay.W)
    y = oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, 0.1)
    rng = np.random.default_rng(0)
    t = rng.integers(0, 7, 50)
    n = rng.integers(0, 48, 50)
    ys = oracle.forward_sampled(x, codes, s, z, lay.A, lay.B, lay.wg, 0.1, t, n)
    assert np.array_equal(ys, y[t, n])


def test_prefill_recipe_opens_about_30_percent_of_gates():
    lay = make_layer(4096, 8, 64, seed=0, gate_open_frac=0.3)
    x = make_x(2048, 4096, seed=0)
    g = oracle.gate(x, lay.wg, lay.b_g)
    frac = float(np.mean(g > 0.5))
    assert 0.25 <= frac <= 0.35, frac


# ------------------------------------------------------------------ planted mistakes

MUTANTS = {
    "drop_ec_term": ("y[t * N + n] = main_part + corr;", "y[t * N + n] = main_part;"),
    "zero_point_sign": ("- (int)z[n])", "+ (int)z[n])"),
    "B_transposed": ("B[(int64_t)j * N + n]", "B[(int64_t)n * r + j]"),
    "A_transposed": ("A[k * r + j]", "A[(int64_t)j * K + k]"),
    "gate_sign": ("exp(-logit)", "exp(logit)"),
    "gate_bias_dropped": ("logit += b_g;", ";"),
    "nibble_order": ("<< (4 * i)", "<< (4 * (7 - i))"),
    "ties_away_from_zero": ("nearbyint((double)quot)", "round((double)quot)"),
    "scale_over_8": ("amax / 7.0", "amax / 8.0"),
    "fp64_scale_in_quotient": ("/ (double)sn)", "/ (amax / 7.0))"),
    "asym_range_over_16": ("(double)range / 15.0", "(double)range / 16.0"),
    "asym_zero_point_sign": ("(-lo / (double)sa)", "(lo / (double)sa)"),
    "asym_zero_not_in_range": ("double lo = 0.0, hi = 0.0;", "double lo = 1e300, hi = -1e300;"),
    "asym_ties_away_from_zero": ("nearbyint((double)qt)", "round((double)qt)"),
    "asym_fp64_quotient": ("float qt = (float)(bf16_to_f64(row[8 * j + i]) / (double)sa);",
                           "double qt = bf16_to_f64(row[8 * j + i]) / (double)sa;"),
}


def _compile_mutant(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    assert old in src, f"mutation site for {name} not found"
    mut = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(mut)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-std=c11", "-o", str(so), str(c), "-lm"])
    return oracle.load_from(str(so))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    lib = _compile_mutant(tmp_path, name, old, new)
    caught = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin fails on the planted mistake '{name}'"
