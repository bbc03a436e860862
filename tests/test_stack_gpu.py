"""A 1B-class decoder's linears as W4 layers, ECs on four seeded layers.

Hidden 2048, intermediate 8192, 16 layers, 7 projections per layer
(q, o: 2048x2048; k, v: 2048->512; gate, up: 2048->8192; down: 8192->2048),
all W4 per output channel, rank-32 ECs on the projections of 4 seeded
layers (the placement the pages' diagnostic would choose is an input here).
A decode pass at M = 64 and a prefill pass at M = 1024 chain outputs into
inputs: q, k, v = P(h); o = P_o(q); gate, up = P(o); down = P_down(up); the
next h = down.  Every linear is checked against the oracle fed the GPU's own
bf16 input, on sampled outputs (tolerance as in tests/helpers.py).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close
from w4_gemm_error_b200.inputs import STACK_1B, STACK_1B_PROJ, make_layer, make_x, stack_ec_layers

pytestmark = pytest.mark.gpu


def test_layer_stack_decode_then_prefill():
    from w4_gemm_error_b200.spear import W4ECLinear
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
        for M in Ms:
            h = hs[M]
            outs = {}

            def run(name, x):
                lin, lay, (codes, s, z) = lins[name]
                y = lin(x)
                torch.cuda.synchronize()
                assert lin.status() == 0
                t = rng.integers(0, M, 128)
                n = rng.integers(0, lay.W.shape[0], 128)
                ref = oracle.forward_sampled(x.cpu(), codes, s, z, lay.A, lay.B, lay.wg, lay.b_g, t, n)
                assert_close(y.float().cpu()[t, n], ref, f"layer {layer} {name} M={M}")
                assert torch.isfinite(y).all()
                return y

            for name in ("q", "k", "v"):
                outs[name] = run(name, h)
            outs["o"] = run("o", outs["q"])
            outs["gate"] = run("gate", outs["o"])
            outs["up"] = run("up", outs["o"])
            outs["down"] = run("down", outs["up"])
            hs[M] = outs["down"]
            checked += 7
        for lin, _, _ in lins.values():
            lin.close()
    assert checked == cfg["layers"] * 7 * len(Ms)
