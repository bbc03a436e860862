"""Layer stacks through the C ABI (spear_w4ec_stack_*), against the oracle.

A 1B-class decoder's linears as W4 layers, ECs on four seeded layers:
hidden 2048, intermediate 8192, 16 layers, 7 projections per layer (q, o:
2048x2048; k, v: 2048->512; gate, up: 2048->8192; down: 8192->2048), all W4
per output channel, rank-32 ECs on the projections of 4 seeded layers (the
placement the pages' diagnostic would choose is an input here).  Each decoder
layer is one stack of 7 ops: q, k, v = P(h); o = P_o(q); gate, up = P(o);
down = P_down(up), and the next layer's h is down.  A decode pass at M = 64
and a prefill pass at M = 1024 run through all 16 layers; every op's output
(read back from the stack's buffers) is checked against the oracle fed the
GPU's own bf16 input, on four outputs of every output tile (tolerance as in
tests/helpers.py).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from helpers import Problem, assert_close, per_tile_samples, tc_token_tile
from w4_gemm_error_b200.inputs import STACK_1B, STACK_1B_PROJ, make_layer, make_x, stack_ec_layers

pytestmark = pytest.mark.gpu

# op name -> (input buffer, output buffer); 0 = h, 1 = the layer's output (down)
DECODER_OPS = {"q": (0, 2), "k": (0, 3), "v": (0, 4), "o": (2, 5), "gate": (5, 6), "up": (5, 7),
               "down": (7, 1)}


def test_layer_stack_decode_then_prefill():
    from w4_gemm_error_b200.spear import W4ECLinear, W4ECStack
    cfg = STACK_1B
    ec_layers = set(stack_ec_layers(0, cfg["layers"], cfg["ec_layers"]))
    assert len(ec_layers) == 4
    Ms = (cfg["decode_M"], cfg["prefill_M"])
    hs = {M: make_x(M, cfg["hidden"], seed=0).cuda() for M in Ms}
    rng = np.random.default_rng(0)
    checked = 0
    for layer in range(cfg["layers"]):
        r = cfg["r"] if layer in ec_layers else 0
        lins = {}
        for p, (name, K, N) in enumerate(STACK_1B_PROJ):
            lay = make_layer(K, N, r, seed=1000 + 7 * layer + p)
            lin = W4ECLinear(lay.W.cuda(), lay.A.cuda() if r else None, lay.B.cuda() if r else None,
                             lay.wg.cuda() if r else None, lay.b_g, max_M=max(Ms))
            lins[name] = (lin, lay, oracle.pack(lay.W))
        stack = W4ECStack([(lins[name][0], i, o, 1) for name, (i, o) in DECODER_OPS.items()], max(Ms))
        for M in Ms:
            h = hs[M]
            y = stack(h)
            torch.cuda.synchronize()
            for lin, _, _ in lins.values():
                assert lin.status() == 0
            bufs = {0: h, 1: y}
            for b in range(2, 8):
                bufs[b] = stack.buffer(b, M)
            for name, (i, o) in DECODER_OPS.items():
                lin, lay, (codes, s, z) = lins[name]
                x_in, out = bufs[i], bufs[o]
                # four outputs of every 128-row output tile of the tcgen05
                # kernel (both batch sizes take it), by index
                t, n = per_tile_samples(M, lay.W.shape[0], tc_token_tile(M), seed=int(rng.integers(1 << 30)))
                ref = oracle.forward_sampled(x_in.cpu(), codes, s, z, lay.A, lay.B, lay.wg, lay.b_g, t, n)
                assert_close(out.float().cpu()[t, n], ref, f"layer {layer} {name} M={M}")
                assert torch.isfinite(out).all()
                checked += 1
            hs[M] = y
        stack.close()
        for lin, _, _ in lins.values():
            lin.close()
    assert checked == cfg["layers"] * 7 * len(Ms)


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_chained_stack_equals_layer_by_layer_forwards(M):
    """A chain of six square layers with ECs placed on layers 1 and 4 only:
    the stack's output (device and host-buffer calls, eager and inside a CUDA
    graph) is bit for bit that of six spear_w4ec_forward calls with flags 0
    on the placed layers and SPEAR_EC_OFF on the others; the last layer's
    output also matches the oracle applied to the input it received."""
    from w4_gemm_error_b200 import spear
    from w4_gemm_error_b200.spear import W4ECStack
    K = 1024
    probs = [Problem(M, K, K, 32, seed=40 + i) for i in range(6)]
    placed = {1, 4}
    ops = []
    for i, P in enumerate(probs):
        ops.append((P.lin, 0 if i == 0 else 2 + (i - 1) % 2, 1 if i == 5 else 2 + i % 2, int(i in placed)))
    stack = W4ECStack(ops, max_M=M)
    x = probs[0].xd
    y = stack(x)
    torch.cuda.synchronize()
    # reference: the same layers, one forward call each
    xs = [x]
    for i, P in enumerate(probs):
        xs.append(P.lin(xs[-1], 0 if i in placed else spear.SPEAR_EC_OFF))
    torch.cuda.synchronize()
    assert torch.equal(y, xs[-1])
    # host buffers
    x_h = probs[0].x.clone().pin_memory()
    y_h = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
    stack.forward_host(x_h, y_h)
    assert torch.equal(y_h, xs[-1].cpu())
    # captured in a CUDA graph on a side stream
    st = torch.cuda.Stream()
    y_g = torch.empty_like(y)
    with torch.cuda.stream(st):
        stack.forward(x, out=y_g, stream=st)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            stack.forward(x, out=y_g, stream=st)
        y_g.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y_g, xs[-1])
    # the last layer against the oracle, on the input it received
    P = probs[5]
    codes, s_, z_ = P.oracle_packed()
    L = P.layer
    ref = oracle.forward(xs[5].cpu(), codes, s_, z_, L.A, L.B, L.wg, L.b_g, ec_on=False)
    assert_close(y, ref, "last layer (EC not placed)")
    stack.close()
    for P in probs:
        P.close()


def test_stack_placement_and_buffer_rules():
    """ec = 0 runs a layer with an EC as the plain W4 GEMM (bitwise
    SPEAR_EC_OFF); the stack rejects buffer plans that do not compose."""
    from w4_gemm_error_b200 import spear
    from w4_gemm_error_b200.spear import W4ECStack
    P = Problem(8, 512, 256, 16, seed=50)
    Q = Problem(8, 256, 512, 16, seed=51)
    y_off = P.lin(P.xd, spear.SPEAR_EC_OFF)
    st_off = W4ECStack([(P.lin, 0, 1, 0)], max_M=8)
    st_on = W4ECStack([(P.lin, 0, 1, 1)], max_M=8)
    assert torch.equal(st_off(P.xd), y_off)
    assert torch.equal(st_on(P.xd), P.lin(P.xd))
    assert torch.equal(st_on(P.xd, spear.SPEAR_EC_OFF), y_off)   # a caller-wide EC_OFF
    st_off.close()
    st_on.close()
    bad = [
        [(P.lin, 0, 2, 1), (Q.lin, 3, 1, 1)],     # reads a buffer nothing wrote
        [(P.lin, 0, 1, 1), (Q.lin, 0, 1, 1)],     # only the last op writes y (and K differs)
        [(P.lin, 0, 2, 1), (P.lin, 2, 1, 1)],     # P reads 256-wide activations as K = 512
        [(P.lin, 0, 2, 1), (Q.lin, 2, 2, 1)],     # reads the buffer it writes
        [(P.lin, 1, 2, 1)],                       # reads y
    ]
    for ops in bad:
        with pytest.raises(spear.SpearError) as ei:
            W4ECStack(ops, max_M=8)
        assert ei.value.status == spear.SPEAR_ERR_INVALID, ops
    with pytest.raises(spear.SpearError) as ei:
        W4ECStack([(P.lin, 0, 1, 1)], max_M=9)     # beyond the layer's max_M
    assert ei.value.status == spear.SPEAR_ERR_INVALID
    ok = W4ECStack([(P.lin, 0, 2, 1), (Q.lin, 2, 1, 1)], max_M=8)
    y = ok(P.xd)
    torch.cuda.synchronize()
    assert torch.equal(y, Q.lin(P.lin(P.xd)))
    ok.close()
    P.close()
    Q.close()
