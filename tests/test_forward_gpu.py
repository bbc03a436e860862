"""Forward pass through the C ABI vs the fp64 oracle, plus bitwise invariants.

Tolerance: see tests/helpers.py (elementwise 1e-2 + 1e-2*|y_ref|, relative
Frobenius 5e-3).  Configurations follow the Llama-class shapes of the
workloads (tiny 16x256x256 r8, q/o 4096x4096 r32, MLP 4096x14336 and
14336x4096 r64, prefill 4096x14336 r64).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from helpers import Problem, assert_close, per_tile_samples, tc_token_tile

pytestmark = pytest.mark.gpu

FUSED, SPLIT, DECODE, TC, EC_OFF = 2, 4, 8, 16, 1


def _run(P: Problem, flags=0, x=None):
    torch.cuda.synchronize()
    y = P.lin(P.xd if x is None else x, flags)
    torch.cuda.synchronize()
    assert P.lin.status() == 0
    return y


@pytest.mark.parametrize("M", [1, 2, 5, 8, 13, 16])
def test_tiny_config_all_token_counts(M):
    P = Problem(M, 256, 256, 8, seed=0, x_outlier_frac=0.0)
    assert_close(_run(P), P.oracle_y())
    P.close()


@pytest.mark.parametrize("M,K,N,r", [(3, 136, 40, 5), (33, 200, 72, 3), (17, 1032, 264, 20), (40, 64, 8, 1),
                                     (7, 8, 8, 1), (9, 4104, 136, 33)])
def test_ragged_shapes(M, K, N, r):
    P = Problem(M, K, N, r, seed=M + K)
    for flags in (0, DECODE | FUSED, DECODE | SPLIT):
        assert_close(_run(P, flags), P.oracle_y(), f"flags={flags}")
    P.close()


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_qo_full_size(M):
    P = Problem(M, 4096, 4096, 32, seed=0)
    ref = P.oracle_y()
    assert_close(_run(P), ref)
    assert_close(_run(P, DECODE | SPLIT), ref, "split")
    P.close()


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
@pytest.mark.parametrize("M", [1, 16])
def test_decode_mlp_full_size(M, K, N):
    P = Problem(M, K, N, 64, seed=0)
    assert_close(_run(P), P.oracle_y())
    P.close()


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
@pytest.mark.parametrize("M", [64, 128])
def test_decode_mlp_larger_batches_sampled(M, K, N):
    P = Problem(M, K, N, 64, seed=0)
    y = _run(P).cpu()
    # four outputs of every output tile (the tcgen05 kernel's 128 rows x
    # 64 / 128 tokens), by index, and 1000 random ones
    t, n = per_tile_samples(M, N, tc_token_tile(M), seed=M)
    rng = np.random.default_rng(M)
    t = np.concatenate([t, rng.integers(0, M, 1000)])
    n = np.concatenate([n, rng.integers(0, N, 1000)])
    assert_close(y.float()[t, n], P.oracle_sampled(t, n))
    P.close()


# Decode kernel with K split over a cluster (up to 16 tokens, K >= 512):
# shapes chosen to reach its corners.  1032 x 264: K split in two with an odd
# chunk count (the ranks hold 3 and 2 chunks, one stage of a single chunk);
# 14336 x 4096: eight-way split with 7 chunks per rank and two EC units per
# CTA (both G buffers cycle); 2048 x 8192: four groups of tiles per cluster;
# 4096 x 1000: ragged rows, two token groups; 8192 x 2048 without an EC;
# 4096 x 14336 at rank 128: nine 16-row groups of G (the most it takes).
@pytest.mark.parametrize("M,K,N,r", [(5, 1032, 264, 20), (16, 14336, 4096, 64), (3, 2048, 8192, 32),
                                     (12, 4096, 1000, 48), (1, 8192, 2048, 0), (9, 4096, 14336, 128)])
def test_cluster_split_decode_shapes(M, K, N, r, monkeypatch):
    monkeypatch.setenv("SPEAR_DECODE_STREAM", "1")
    P = Problem(M, K, N, r, seed=M + K + N)
    ref = P.oracle_y()
    flag_sets = (DECODE | FUSED, DECODE | SPLIT) if r else (DECODE | FUSED,)
    for flags in flag_sets:
        assert_close(_run(P, flags), ref, f"flags={flags}")
    assert_close(_run(P, DECODE | EC_OFF), P.oracle_y(ec_on=False), "EC off")
    y1 = _run(P, DECODE | FUSED)
    assert torch.equal(_run(P, DECODE | FUSED), y1), "repeated runs differ"
    P.close()


def test_ec_isolated_on_qo_shape():
    """y(EC on) - y(EC off) against the oracle's correction term alone."""
    P = Problem(16, 4096, 4096, 32, seed=3)
    y_on = _run(P).double().cpu().numpy()
    y_off = _run(P, EC_OFF).double().cpu().numpy()
    ref_on, g, corr = P.oracle_y(want_corr=True)
    ref_off = ref_on - corr
    delta = y_on - y_off
    # Error budget of delta - corr, element by element: the two bf16 roundings
    # of y (unit roundoff 2^-8 each) and the fp32 evaluation of the correction
    # (u = x.A accumulated in fp32 from exact bf16 products, then g_t and
    # sum_j u_j B_j in fp32: far below 1e-4 of sum_j |u_j B_j|); the main
    # product is computed the same way with and without the EC, so its fp32
    # error cancels.  No operand of the correction is rounded to bf16.
    xd = P.x.double().numpy()
    terms = g[:, None] * (np.abs(xd @ P.layer.A.double().numpy()) @ np.abs(P.layer.B.double().numpy()))
    bound = 2.0 ** -8 * (np.abs(ref_on) + np.abs(ref_off)) + 1e-4 * terms + 1e-6
    assert np.all(np.abs(delta - corr) <= bound)
    # in aggregate the difference tracks the correction (bf16 rounding of y
    # alone leaves about 10% relative noise at this correction size)
    assert np.linalg.norm(delta - corr) / np.linalg.norm(corr) < 0.25
    P.close()


def test_ec_dominant_variant():
    """A, B ~ N(0, 1): the correction dominates y, so y's tolerance checks the EC.

    The fused decode kernel keeps v = g*(x.A) in fp32 and meets the plain
    tolerance.  The split path rounds the plain GEMM's output to bf16 before
    adding the correction (2^-8 of |main| more where main and correction
    cancel); the tcgen05 kernel feeds v and B^T/s to the tensor cores as
    tf32 (up to 2^-11 of |v_j B_j| per term for each of the two roundings).
    Their bounds add those terms to the plain tolerance.
    """
    P = Problem(16, 4096, 4096, 32, seed=4, ab_std=1.0)
    ref, g, corr = P.oracle_y(want_corr=True)
    assert np.linalg.norm(corr) > 10 * np.linalg.norm(ref - corr)
    assert_close(_run(P), ref)
    y_split = _run(P, DECODE | SPLIT).double().cpu().numpy()
    assert np.all(np.abs(y_split - ref) <= 1e-2 + 1e-2 * np.abs(ref) + 2.0 ** -8 * np.abs(ref - corr))
    xd = P.x.double().numpy()
    terms = g[:, None] * (np.abs(xd @ P.layer.A.double().numpy()) @ np.abs(P.layer.B.double().numpy()))
    y_tc = _run(P, TC | FUSED).double().cpu().numpy()
    assert np.all(np.abs(y_tc - ref) <= 1e-2 + 1e-2 * np.abs(ref) + 2.0 ** -10 * terms)
    assert np.linalg.norm(y_tc - ref) / np.linalg.norm(ref) < 5e-3
    P.close()


def test_gate_matches_oracle():
    P = Problem(37, 4096, 256, 64, seed=5, gate_open_frac=0.3)
    g = P.lin.gate(P.xd).double().cpu().numpy()
    import oracle
    g_ref = oracle.gate(P.x, P.layer.wg, P.layer.b_g)
    assert np.max(np.abs(g - g_ref)) < 1e-5
    P.close()


def test_gate_closed_and_open_limits():
    P = Problem(8, 512, 64, 8, seed=6)
    y_lin = _run(P, EC_OFF)
    P.lin.close()
    from w4_gemm_error_b200.spear import W4ECLinear
    L = P.layer
    closed = W4ECLinear(L.W.cuda(), L.A.cuda(), L.B.cuda(), L.wg.cuda(), -1e4, max_M=8)
    assert torch.equal(closed(P.xd), y_lin)          # g == 0 exactly: the plain W4 GEMM
    closed.close()


def test_ec_off_equals_zero_B_and_rank_zero():
    P = Problem(12, 1024, 384, 16, seed=7)
    y_off = _run(P, EC_OFF)
    from w4_gemm_error_b200.spear import W4ECLinear
    L = P.layer
    zb = W4ECLinear(L.W.cuda(), L.A.cuda(), torch.zeros_like(L.B).cuda(), L.wg.cuda(), L.b_g, max_M=12)
    r0 = W4ECLinear(L.W.cuda(), None, None, None, 0.0, max_M=12)
    assert torch.equal(zb(P.xd), y_off)
    assert torch.equal(r0(P.xd), y_off)
    zb.close()
    r0.close()
    P.close()


def test_invariants_determinism_scaling_permutation():
    P = Problem(16, 4096, 1024, 32, seed=8)
    y1 = _run(P)
    for _ in range(3):
        assert torch.equal(_run(P), y1), "repeated runs differ"
    y_off = _run(P, EC_OFF)
    y2 = _run(P, EC_OFF, x=(P.xd.float() * 2).to(torch.bfloat16))
    assert torch.equal(y2, (y_off.float() * 2).to(torch.bfloat16)), "y(2x) != 2 y(x)"
    perm = torch.randperm(16, generator=torch.Generator().manual_seed(0))
    yp = _run(P, 0, x=P.xd[perm.cuda()].contiguous())
    assert torch.equal(yp, y1[perm.cuda()]), "token permutation"
    P.close()


@pytest.mark.parametrize("M,K,N,r", [(1, 4096, 4096, 32), (16, 4096, 4096, 32), (24, 4096, 4096, 32),
                                     (1, 4096, 14336, 64), (5, 1032, 264, 20)])
def test_prefetch_hint_leaves_results_unchanged(M, K, N, r):
    """The cross-layer prefetch hint only moves weights into L2: a chain of
    layers that name each other (and one that names itself) gives bitwise the
    same outputs as the same chain without hints; destroying a named layer
    clears the hint of the layer that names it."""
    P = Problem(M, K, N, r, seed=M + N)
    Q = Problem(M, K, N, r, seed=M + N + 1)
    ref_p, ref_q = _run(P), _run(Q)
    P.lin.set_next(Q.lin)
    Q.lin.set_next(P.lin)
    for _ in range(2):
        assert torch.equal(_run(P), ref_p)
        assert torch.equal(_run(Q), ref_q)
    Q.lin.set_next(Q.lin)
    assert torch.equal(_run(Q), ref_q)
    Q.close()
    assert torch.equal(_run(P), ref_p)   # P's hint was cleared with Q
    P.close()


@pytest.mark.parametrize("M,K,N,r", [(1, 4096, 4096, 32), (4, 4096, 4096, 32), (16, 4096, 4096, 32),
                                     (1, 4096, 14336, 64)])
def test_alternating_inputs_and_layers(M, K, N, r):
    """Forwards whose inputs change from call to call, interleaved over two
    layers: each output must match the oracle for its own input, so no EC
    value or partial product left in shared or global memory by an earlier
    forward (of this layer or another) can stand in for the current one."""
    import oracle as orc
    from w4_gemm_error_b200.inputs import make_x
    P = Problem(M, K, N, r, seed=3)
    Q = Problem(M, K, N, r, seed=4)
    xs = [make_x(M, K, seed=100 + i) for i in range(3)]
    refs = {}
    for name, prob in (("P", P), ("Q", Q)):
        codes, s_, z = prob.oracle_packed()
        L = prob.layer
        refs[name] = [orc.forward(x, codes, s_, z, L.A, L.B, L.wg, L.b_g) for x in xs]
    for rnd in range(2):
        for i, x in enumerate(xs):
            for name, prob in (("P", P), ("Q", Q)):
                y = _run(prob, 0, x=x.cuda())
                assert_close(y, refs[name][i], f"{name} input {i} round {rnd}")
    P.close()
    Q.close()


@pytest.mark.parametrize("M", [1, 4, 16, 24, 64])
def test_chained_layers_on_one_stream(M):
    """Four square layers chained on one stream with no host synchronisation
    in between (each kernel starts early through programmatic dependent launch
    and waits for its input on the device), in a captured CUDA graph as the
    bench runs them: every layer's output matches the oracle applied to the
    input that layer actually received."""
    import oracle as orc
    from w4_gemm_error_b200.inputs import make_layer
    from w4_gemm_error_b200.spear import W4ECLinear
    K = 1024
    layers, lins = [], []
    for i in range(4):
        L = make_layer(K, K, 32, seed=20 + i)
        layers.append(L)
        lins.append(W4ECLinear(L.W.cuda(), L.A.cuda(), L.B.cuda(), L.wg.cuda(), L.b_g, max_M=M))
    for i in range(4):
        lins[i].set_next(lins[(i + 1) % 4])
    P0 = Problem(M, K, K, 32, seed=30)
    st = torch.cuda.Stream()
    ys = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in range(4)]

    def chain():
        x = P0.xd
        for i in range(4):
            lins[i].forward(x, 0, out=ys[i], stream=st)
            x = ys[i]

    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        chain()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            chain()
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    for lin in lins:
        assert lin.status() == 0
    x_in = P0.x
    for i in range(4):
        codes, s_, z = orc.pack(layers[i].W)
        L = layers[i]
        ref = orc.forward(x_in, codes, s_, z, L.A, L.B, L.wg, L.b_g)
        assert_close(ys[i], ref, f"layer {i}")
        x_in = ys[i].cpu()
    for lin in lins:
        lin.close()
    P0.close()


def test_host_buffer_entry_matches_device_entry():
    from w4_gemm_error_b200 import spear
    P = Problem(9, 1024, 512, 16, seed=9)
    y_dev = _run(P).cpu()
    x_h = P.x.clone().pin_memory()
    y_h = torch.empty((9, 512), dtype=torch.bfloat16).pin_memory()
    spear.spear_w4ec_forward_host(P.lin.h, x_h, y_h, 9)
    assert torch.equal(y_h, y_dev)
    P.close()


def test_tune_records_a_legal_choice():
    P = Problem(16, 4096, 4096, 32, seed=10)
    y = torch.empty((16, 4096), dtype=torch.bfloat16, device="cuda")
    choice = P.lin.tune(P.xd, y)
    assert choice & (DECODE | TC) and choice & (FUSED | SPLIT)
    assert P.lin.dispatch(16) == choice
    assert_close(_run(P), P.oracle_y())
    P.close()


def test_argument_errors():
    from w4_gemm_error_b200 import spear
    P = Problem(4, 256, 256, 8, seed=11, max_M=4)
    h = P.lin.h
    lib = spear.lib()
    y = torch.empty((8, 256), dtype=torch.bfloat16, device="cuda")
    x8 = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert lib.spear_w4ec_forward(h, x8.data_ptr(), y.data_ptr(), 8, 0, s) == spear.SPEAR_ERR_INVALID  # M > max_M
    assert lib.spear_w4ec_forward(h, x8.data_ptr() + 2, y.data_ptr(), 1, 0, s) == spear.SPEAR_ERR_INVALID
    assert lib.spear_w4ec_forward(h, x8.data_ptr(), y.data_ptr(), 0, 0, s) == spear.SPEAR_OK
    assert lib.spear_w4ec_forward(h, x8.data_ptr(), y.data_ptr(), 1, DECODE | TC, s) == spear.SPEAR_ERR_INVALID
    fresh = spear.spear_w4ec_create(256, 256, 8, 4)
    assert lib.spear_w4ec_forward(fresh, x8.data_ptr(), y.data_ptr(), 1, 0, s) == spear.SPEAR_ERR_STATE
    spear.spear_w4ec_destroy(fresh)
    r0 = spear.spear_w4ec_create(256, 256, 0, 4)
    g = torch.empty(4, device="cuda")
    assert lib.spear_w4ec_get_gate(r0, x8.data_ptr(), g.data_ptr(), 1, s) == spear.SPEAR_ERR_UNSUPPORTED
    spear.spear_w4ec_destroy(r0)
    P.close()


def test_injected_faults_are_reported(monkeypatch):
    from w4_gemm_error_b200 import spear
    monkeypatch.setenv("SPEAR_FAULT", "alloc")
    with pytest.raises(spear.SpearError) as ei:
        spear.spear_w4ec_create(256, 256, 8, 4)
    assert ei.value.status == spear.SPEAR_ERR_NOMEM
    monkeypatch.setenv("SPEAR_FAULT", "launch")
    P = Problem(4, 256, 256, 8, seed=12)
    with pytest.raises(spear.SpearError) as ei:
        P.lin(P.xd)
    assert ei.value.status == spear.SPEAR_ERR_CUDA
    P.close()
    # a tcgen05 launch that reports a timeout (its prepass has run and counted
    # v): the status says so, and the handle's counters are cleared for later
    monkeypatch.setenv("SPEAR_FAULT", "timeout")
    P = Problem(64, 512, 256, 8, seed=13)
    for _ in range(2):
        torch.cuda.synchronize()
        P.lin(P.xd, TC | FUSED)
        assert P.lin.status() == spear.SPEAR_ERR_TIMEOUT
    P.close()


# ------------------------------------------------------------------ tcgen05 tile kernel

# token tiles of 32 (M <= 32), 64, 128 and 256 columns
@pytest.mark.parametrize("M,K,N,r", [(33, 256, 128, 8), (256, 4096, 1024, 64), (300, 512, 256, 32),
                                     (1000, 1032, 264, 20), (513, 4104, 136, 33), (64, 2048, 512, 32),
                                     (9, 8, 8, 1), (700, 8192, 256, 128), (100, 1032, 264, 20),
                                     (128, 512, 384, 16), (32, 4096, 256, 64)])
def test_tc_path_shapes(M, K, N, r):
    P = Problem(M, K, N, r, seed=M + N)
    ref = P.oracle_y()
    for flags in (TC | FUSED, TC | SPLIT):
        assert_close(_run(P, flags), ref, f"flags={flags}")
    assert_close(_run(P, TC | EC_OFF), P.oracle_y(ec_on=False), "EC off")
    P.close()


# Persistent tcgen05 kernel with more output tiles than CTAs (148 SMs): each
# CTA runs two or three tiles in turn, alternating its two TMEM accumulators,
# reusing them across tiles and carrying the shared-memory ring's phase from
# one tile to the next.  Every output is compared with the oracle.
#   1024 x 8192: 4 token tiles x 64 row tiles = 256 tiles
#   600 x 14336: 3 token tiles (the last one ragged, 88 tokens) x 112 = 336 tiles
@pytest.mark.parametrize("M,K,N,r", [(1024, 1024, 8192, 32), (600, 512, 14336, 16)])
def test_tc_persistent_tiles_full_output(M, K, N, r):
    P = Problem(M, K, N, r, seed=M + 1)
    tiles = -(-M // tc_token_tile(M)) * (N // 128)
    assert tiles > torch.cuda.get_device_properties(0).multi_processor_count
    ref = P.oracle_y()
    for flags in (TC | FUSED, TC | SPLIT):
        assert_close(_run(P, flags), ref, f"flags={flags}")
    assert_close(_run(P, TC | EC_OFF), P.oracle_y(ec_on=False), "EC off")
    P.close()


# Split K at its widest: a layer of 16 row tiles splits every tile's K into
# min(8, SMs / tiles) = 8 units (128 units on 148 CTAs; the split is sized so
# that the units never outnumber the SMs), the last unit of each tile summing
# the partials in split order.  Full outputs, ragged N and ragged tokens.
@pytest.mark.parametrize("M,K,N,r", [(128, 4096, 2048, 64), (37, 4096, 2000, 32)])
def test_tc_split_k_eight_ways_full_output(M, K, N, r):
    P = Problem(M, K, N, r, seed=M + 2)
    ref = P.oracle_y()
    for flags in (TC | FUSED, TC | SPLIT):
        assert_close(_run(P, flags), ref, f"flags={flags}")
    assert_close(_run(P, TC | EC_OFF), P.oracle_y(ec_on=False), "EC off")
    P.close()


def test_tc_path_invariants():
    P = Problem(300, 1024, 512, 32, seed=13)
    y1 = _run(P, TC)
    assert torch.equal(_run(P, TC), y1), "repeated runs differ"
    y_off = _run(P, TC | EC_OFF)
    y2 = _run(P, TC | EC_OFF, x=(P.xd.float() * 2).to(torch.bfloat16))
    assert torch.equal(y2, (y_off.float() * 2).to(torch.bfloat16)), "y(2x) != 2 y(x)"
    perm = torch.randperm(300, generator=torch.Generator().manual_seed(1))
    yp = _run(P, TC, x=P.xd[perm.cuda()].contiguous())
    assert torch.equal(yp, y1[perm.cuda()]), "token permutation"
    P.close()


def test_tc_split_k_invariants():
    # a narrow layer (4 row tiles) at 64 tokens: K split four ways, partials summed
    # by the last unit of each tile in split order, so runs are bit-identical
    P = Problem(64, 2048, 512, 32, seed=15)
    y1 = _run(P, TC)
    for _ in range(3):
        assert torch.equal(_run(P, TC), y1), "repeated split-K runs differ"
    y_off = _run(P, TC | EC_OFF)
    y2 = _run(P, TC | EC_OFF, x=(P.xd.float() * 2).to(torch.bfloat16))
    assert torch.equal(y2, (y_off.float() * 2).to(torch.bfloat16)), "y(2x) != 2 y(x)"
    perm = torch.randperm(64, generator=torch.Generator().manual_seed(2))
    yp = _run(P, TC, x=P.xd[perm.cuda()].contiguous())
    assert torch.equal(yp, y1[perm.cuda()]), "token permutation"
    assert_close(y1, P.oracle_y(), "split-K vs oracle")
    P.close()


def test_tc_ec_isolated():
    P = Problem(256, 4096, 1024, 64, seed=14)
    y_on = _run(P, TC).double().cpu().numpy()
    y_off = _run(P, TC | EC_OFF).double().cpu().numpy()
    ref_on, g, corr = P.oracle_y(want_corr=True)
    ref_off = ref_on - corr
    xd = P.x.double().numpy()
    terms = g[:, None] * (np.abs(xd @ P.layer.A.double().numpy()) @ np.abs(P.layer.B.double().numpy()))
    # two bf16 roundings of y, and the tf32 operands v and B^T/s of the EC
    bound = 2.0 ** -8 * (np.abs(ref_on) + np.abs(ref_off)) + 2.0 ** -10 * terms + 1e-4 * terms + 1e-6
    assert np.all(np.abs((y_on - y_off) - corr) <= bound)
    P.close()


@pytest.mark.parametrize("M", [2048, 4096])
def test_prefill_full_size_sampled(M):
    """Prefill MLP gate/up shape, heavy rows and ~30% open gates: four outputs
    of every 128-row x 256-token output tile (896 and 1792 tiles, so every
    persistent CTA's second and later tiles are among them), by index."""
    P = Problem(M, 4096, 14336, 64, seed=0, w_row_outlier_frac=0.005, gate_open_frac=0.3)
    y = _run(P).float().cpu()
    t, n = per_tile_samples(M, 14336, tc_token_tile(M), seed=M)
    assert len(t) == 4 * (M // 256) * 112
    assert_close(y[t, n], P.oracle_sampled(t, n))
    # every row of y is finite and the gate opened for about 30% of tokens
    assert torch.isfinite(y).all()
    g = P.lin.gate(P.xd).cpu().numpy()
    assert 0.25 <= float(np.mean(g > 0.5)) <= 0.35
    P.close()
