"""The persistent stack kernel (spear_w4ec_stack_forward with
SPEAR_STACK_PERSISTENT) against the oracle.

One launch runs every op of the stack; each op's output is read back (the
stack's buffers) and compared with the fp64 oracle fed that op's own bf16
input as the GPU saw it, elementwise and in Frobenius norm (tolerance as in
tests/helpers.py).  The graphs cover every way an op gets its EC input:
  * ops that read the stack's input, or a buffer written earlier than by the
    op just before (EC down-projection by the op's own EC units),
  * ops that read the previous op's output (u formed in that op's epilogue),
  * ops with the EC not placed, layers without an EC, rank 64 (the largest
    the kernel takes), ragged K and N, K not a multiple of 1024;
and the waits: read-after-write chains, and writes to a buffer that an
earlier op wrote or read (a fan of ops reading x into two alternating
buffers).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_close
from w4_gemm_error_b200.inputs import make_layer, make_x

pytestmark = pytest.mark.gpu

PERSIST = 32   # SPEAR_STACK_PERSISTENT


def _layers(shapes, seed):
    """shapes: [(K, N, r)]; returns [(W4ECLinear, layer, packed)]."""
    from w4_gemm_error_b200.spear import W4ECLinear
    out = []
    for i, (K, N, r) in enumerate(shapes):
        lay = make_layer(K, N, r, seed=seed + i)
        lin = W4ECLinear(lay.W.cuda(), lay.A.cuda() if r else None, lay.B.cuda() if r else None,
                         lay.wg.cuda() if r else None, lay.b_g, max_M=16)
        out.append((lin, lay, oracle.pack(lay.W)))
    return out


def _check_ops(stack, layers, ops, x, y, M, ec_on_all=True, what=""):
    """Compare every op's output with the oracle on the op's own GPU input."""
    bufs = {0: x.cpu(), 1: y.cpu()}
    for _, i, o, _ in ops:
        for b in (i, o):
            if b >= 2 and b not in bufs:
                bufs[b] = stack.buffer(b, M).cpu()
    # a buffer written twice holds the last writer's output: check only the
    # ops whose output and input are still as they left them
    last_writer = {}
    for n, (_, _, o, _) in enumerate(ops):
        last_writer[o] = n
    for n, (li, i, o, ec) in enumerate(ops):
        if last_writer[o] != n:
            continue
        if i >= 2 and any(last_writer.get(i) == m for m in range(n + 1, len(ops))):
            continue
        lin, lay, (codes, s, z) = layers[li]
        ref = oracle.forward(bufs[i], codes, s, z, lay.A, lay.B, lay.wg, lay.b_g,
                             ec_on=bool(ec) and ec_on_all)
        assert_close(bufs[o], ref, f"{what} op {n} (layer {li}, {i}->{o}, ec {ec}) M={M}")


def _run(stack, x, M, flags=PERSIST):
    from w4_gemm_error_b200 import spear
    y = torch.empty((M, stack.out_width), dtype=torch.bfloat16, device="cuda")
    stack.forward(x, flags, out=y)
    torch.cuda.synchronize()
    return y


# A decoder layer's projections: q, k, v read h; o reads q; gate and up read
# o; down reads up.  h 512, kv 128, intermediate 1536; ECs of mixed rank,
# one not placed, one layer without an EC.
DECODER = {"shapes": [(512, 512, 32), (512, 128, 16), (512, 128, 0), (512, 512, 64),
                      (512, 1536, 32), (512, 1536, 48), (1536, 512, 64)],
           "ops": [(0, 0, 2, 1), (1, 0, 3, 1), (2, 0, 4, 1), (3, 2, 5, 1), (4, 5, 6, 0), (5, 5, 7, 1),
                   (6, 7, 1, 1)]}


@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
def test_decoder_graph(M):
    from w4_gemm_error_b200.spear import W4ECStack
    layers = _layers(DECODER["shapes"], seed=7000)
    ops = DECODER["ops"]
    stack = W4ECStack([(layers[li][0], i, o, ec) for li, i, o, ec in ops], 16)
    x = make_x(M, 512, seed=M).cuda()
    y = _run(stack, x, M)
    for lin, _, _ in layers:
        assert lin.status() == 0
    _check_ops(stack, layers, ops, x, y, M, what="decoder")
    # every EC off for the call
    y = _run(stack, x, M, PERSIST | 1)
    _check_ops(stack, layers, ops, x, y, M, ec_on_all=False, what="decoder, EC off")
    stack.close()
    for lin, _, _ in layers:
        lin.close()


# A chain of layers (y of one is x of the next): ragged widths (K not a
# multiple of 1024 or of 64, N not a multiple of 16), the EC on, off and
# absent, rank 64, more tiles than CTAs (N = 4104: 257 tiles).
CHAIN = [(776, 200, 32), (200, 4104, 64), (4104, 1032, 0), (1032, 776, 8), (776, 776, 33), (776, 520, 64)]


@pytest.mark.parametrize("M", [1, 6, 16])
def test_ragged_chain(M):
    from w4_gemm_error_b200.spear import W4ECStack
    layers = _layers(CHAIN, seed=7100)
    n = len(CHAIN)
    ops = [(l, 0 if l == 0 else 2 + (l - 1) % 2, 1 if l == n - 1 else 2 + l % 2, 0 if l == 3 else 1)
           for l in range(n)]
    # buffers 2 and 3 alternate, so each intermediate is overwritten two ops
    # later: check the chain op by op on stacks that end at every op
    x = make_x(M, CHAIN[0][0], seed=M + 1).cuda()
    for end in range(1, n + 1):
        sub = [(li, i, 1 if k == end - 1 else o, ec) for k, (li, i, o, ec) in enumerate(ops[:end])]
        stack = W4ECStack([(layers[li][0], i, o, ec) for li, i, o, ec in sub], 16)
        y = _run(stack, x, M)
        for lin, _, _ in layers:
            assert lin.status() == 0
        _check_ops(stack, layers, sub, x, y, M, what=f"chain[:{end}]")
        stack.close()
    for lin, _, _ in layers:
        lin.close()


def test_fan_of_ops_reading_x():
    """Every op reads x and the outputs alternate between two buffers: each
    op waits only for the op two before it (the last writer of its output)."""
    from w4_gemm_error_b200.spear import W4ECStack
    shapes = [(1024, 2048, 32)] * 5
    layers = _layers(shapes, seed=7200)
    ops = [(l, 0, 1 if l == 4 else 2 + l % 2, 1) for l in range(5)]
    stack = W4ECStack([(layers[li][0], i, o, ec) for li, i, o, ec in ops], 16)
    for M in (1, 16):
        x = make_x(M, 1024, seed=M + 2).cuda()
        y = _run(stack, x, M)
        _check_ops(stack, layers, ops, x, y, M, what="fan")
    stack.close()
    for lin, _, _ in layers:
        lin.close()


def test_graph_replay_and_repeat_calls():
    """Captured in a CUDA graph and replayed (the counters and u
    accumulators are cleared inside the capture), and called again eagerly:
    each result matches the oracle."""
    from w4_gemm_error_b200.spear import W4ECStack
    layers = _layers([(1024, 1024, 32)] * 4, seed=7300)
    ops = [(l, 0 if l == 0 else 2 + (l - 1) % 2, 1 if l == 3 else 2 + l % 2, 1) for l in range(4)]
    stack = W4ECStack([(layers[li][0], i, o, ec) for li, i, o, ec in ops], 16)
    M = 4
    x = make_x(M, 1024, seed=11).cuda()
    y = torch.empty((M, 1024), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        stack.forward(x, PERSIST, out=y, stream=s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            stack.forward(x, PERSIST, out=y, stream=s)
    torch.cuda.synchronize()
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        _check_ops(stack, layers, ops, x, y, M, what="graph")
    del g
    y2 = _run(stack, x, M)
    _check_ops(stack, layers, ops, x, y2, M, what="eager after graph")
    stack.close()
    for lin, _, _ in layers:
        lin.close()


def test_unsupported_cases_are_refused():
    from w4_gemm_error_b200 import spear
    from w4_gemm_error_b200.spear import W4ECStack
    layers = _layers([(512, 512, 16)], seed=7400)
    stack = W4ECStack([(layers[0][0], 0, 1, 1)], 16)
    x = make_x(16, 512, seed=3).cuda()
    for flags in (PERSIST | spear.SPEAR_FORCE_DECODE, PERSIST | spear.SPEAR_FORCE_FUSED):
        with pytest.raises(spear.SpearError) as ei:
            stack.forward(x, flags)
        assert ei.value.status == spear.SPEAR_ERR_UNSUPPORTED
    stack.close()
    # more than 16 tokens
    from w4_gemm_error_b200.spear import W4ECLinear
    lay = make_layer(512, 512, 16, seed=9)
    lin = W4ECLinear(lay.W.cuda(), lay.A.cuda(), lay.B.cuda(), lay.wg.cuda(), lay.b_g, max_M=32)
    st = W4ECStack([(lin, 0, 1, 1)], 32)
    with pytest.raises(spear.SpearError) as ei:
        st.forward(make_x(17, 512, seed=4).cuda(), PERSIST)
    assert ei.value.status == spear.SPEAR_ERR_UNSUPPORTED
    st.close()
    lin.close()
    # rank above 64
    lay = make_layer(512, 512, 65, seed=10)
    lin = W4ECLinear(lay.W.cuda(), lay.A.cuda(), lay.B.cuda(), lay.wg.cuda(), lay.b_g, max_M=16)
    st = W4ECStack([(lin, 0, 1, 1)], 16)
    with pytest.raises(spear.SpearError) as ei:
        st.forward(make_x(2, 512, seed=5).cuda(), PERSIST)
    assert ei.value.status == spear.SPEAR_ERR_UNSUPPORTED
    st.close()
    lin.close()
    for lin, _, _ in layers:
        lin.close()


def test_injected_timeout_is_reported(monkeypatch):
    """With SPEAR_FAULT=timeout the kernel's first wait is for a count that
    nothing reaches: every CTA gives up after its bounded wait (about a
    second), the first op's layer reports SPEAR_ERR_TIMEOUT, and the device
    stays usable."""
    from w4_gemm_error_b200 import spear
    from w4_gemm_error_b200.spear import W4ECStack
    monkeypatch.setenv("SPEAR_FAULT", "timeout")
    layers = _layers([(512, 512, 16), (512, 512, 16)], seed=7500)
    stack = W4ECStack([(layers[0][0], 0, 2, 1), (layers[1][0], 2, 1, 1)], 16)
    _run(stack, make_x(2, 512, seed=6).cuda(), 2)
    assert layers[0][0].status() == spear.SPEAR_ERR_TIMEOUT
    stack.close()
    for lin, _, _ in layers:
        lin.close()
    monkeypatch.delenv("SPEAR_FAULT")
    t = torch.ones(4, device="cuda")
    assert float((t * 2).sum()) == 8.0
