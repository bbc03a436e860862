"""Row-parallel layer (spear_w4ec_tp_*) against the oracle, on one GPU.

The ranks of a group run here as shard handles of one process on one device,
connected with each other's buffer addresses.  Each call issues the partial
phase of every rank and then the reduce phase of every rank on one stream,
so every device wait of a phase is for words that launches before it have
already raised: no kernel waits for a later one.  (On several GPUs the ranks
are processes and the waits are real; their handle exchange is checked here
with two processes that connect and launch nothing.)

Checks, per call:
  * every rank's y is the same, bit for bit (u and the partials are summed
    in rank order on every rank);
  * y against the fp64 oracle of the WHOLE layer: the tolerance of
    tests/helpers.py plus 2^-8 of the sum over ranks of the magnitudes of
    the partial outputs, each of which is rounded to bf16 once before the
    sum (half an ulp is 2^-9 relative; the margin covers the rounding of an
    already rounded value);
  * each rank's partial output against the oracle's plain W4 product of its
    shard (whole-row scales), with the tolerance of tests/helpers.py;
  * each u slot against x_q.[w_g,q, A_q] in fp64, within fp32 accumulation
    (1e-4 of the sum of the products' magnitudes), and every rank holding
    the same slots (the dual write).
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch

import oracle
from helpers import ATOL, FROB, RTOL, assert_close
from w4_gemm_error_b200.inputs import make_layer, make_x

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.float().double().cpu().numpy()


class Group:
    """A layer, its shards over `world` ranks on cuda:0, and the oracle's view."""

    def __init__(self, K, N, r, world, max_M, seed):
        from w4_gemm_error_b200.spear import W4ECLinear, W4ECRowParallel, tp_shard, tp_shard_bounds
        self.lay = lay = make_layer(K, N, r, seed=seed)
        self.K, self.N, self.r, self.world = K, N, r, world
        self.codes, self.s, self.z = oracle.pack(lay.W)
        self.bounds = tp_shard_bounds(K, world)
        codes_d = torch.from_numpy(self.codes.view(np.int32)).cuda()
        s_d = torch.from_numpy(self.s).cuda()
        z_d = torch.from_numpy(self.z).cuda()
        A_d, B_d, wg_d = (lay.A.cuda(), lay.B.cuda(), lay.wg.cuda()) if r else (None, None, None)
        self.shards, self.tps, self.host_shards = [], [], []
        for p, (k0, k1) in enumerate(self.bounds):
            c_p, s_p, z_p, A_p, wg_p = tp_shard(codes_d, s_d, z_d, A_d, wg_d, k0, k1)
            lin = W4ECLinear(None, A_p, B_d, wg_p, lay.b_g, max_M=max_M, packed=(c_p, s_p, z_p))
            self.shards.append(lin)
            self.tps.append(W4ECRowParallel(lin, p, world, max_M))
            self.host_shards.append(tp_shard(self.codes, self.s, self.z, lay.A, lay.wg, k0, k1))
        bases = [t.base for t in self.tps]
        for t in self.tps:
            t.connect(bases)

    def xs(self, x):
        return [x[:, k0:k1].contiguous().cuda() for k0, k1 in self.bounds]

    def call(self, x, flags=0):
        xs = self.xs(x)
        for t, x_p in zip(self.tps, xs):
            t.partial(x_p, flags)
        ys = [t.reduce(x.shape[0], flags) for t in self.tps]
        torch.cuda.synchronize()
        return ys

    def check(self, x, ys, ec_on=True, what=""):
        lay, M = self.lay, x.shape[0]
        for p, y in enumerate(ys[1:], 1):
            assert torch.equal(y, ys[0]), f"{what}: rank {p} differs from rank 0"
        ref = oracle.forward(x, self.codes, self.s, self.z, lay.A, lay.B, lay.wg, lay.b_g, ec_on=ec_on)
        parts = []
        for p, (k0, k1) in enumerate(self.bounds):
            c_p, s_p, z_p, A_p, wg_p = self.host_shards[p]
            x_p = x[:, k0:k1].contiguous()
            ref_p = oracle.forward(x_p, c_p, s_p, z_p, A_p, lay.B, wg_p, lay.b_g, ec_on=False)
            parts.append(ref_p)
            assert_close(self.tps[p].partial_output(M), ref_p, f"{what}: partial output of rank {p}")
        y = _f64(ys[0])
        assert np.all(np.isfinite(y)), what
        extra = 2.0 ** -8 * sum(np.abs(q) for q in parts)
        err = np.abs(y - ref)
        bad = err > ATOL + RTOL * np.abs(ref) + extra
        assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, first at {np.argwhere(bad)[0]}"
        nref = np.linalg.norm(ref)
        if nref > 0:
            assert np.linalg.norm(y - ref) / nref <= FROB + np.linalg.norm(extra) / nref, what
        if ec_on and self.r:
            self.check_slots(x, what)

    def check_slots(self, x, what):
        lay, M = self.lay, x.shape[0]
        slots = [t.u_slots(M).double().cpu().numpy() for t in self.tps]
        for p in range(1, self.world):
            assert np.array_equal(slots[p], slots[0]), f"{what}: rank {p} holds other u slots than rank 0"
        for q, (k0, k1) in enumerate(self.bounds):
            xq = _f64(x[:, k0:k1])
            G = np.concatenate([_f64(lay.wg[k0:k1])[:, None], _f64(lay.A[k0:k1])], axis=1)
            want = xq @ G
            bound = 1e-4 * (np.abs(xq) @ np.abs(G)) + 1e-6
            got = slots[0][q][:, :self.r + 1]
            assert np.all(np.abs(got - want) <= bound), f"{what}: u slot {q}"
            assert not np.any(slots[0][q][:, self.r + 1:]), f"{what}: u slot {q} padding"

    def status(self):
        return [lin.status() for lin in self.shards]

    def close(self):
        for t in self.tps:
            t.close()
        for lin in self.shards:
            lin.close()


@pytest.mark.parametrize("M", [1, 16, 37])
def test_world_of_one_matches_the_oracle(M):
    g = Group(1024, 1032, 32, 1, 40, seed=8000)
    x = make_x(M, 1024, seed=M)
    g.check(x, g.call(x), what=f"world 1 M={M}")
    assert g.status() == [0]
    g.close()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_emulated_ranks(world):
    """Ragged shards (K = 1032 over 2, 3, 4 ranks), N not a multiple of 256,
    rank 33; one, nine and forty tokens (three token blocks of the reduce);
    the EC on and off in alternate calls of the same group."""
    g = Group(1032, 776, 33, world, 40, seed=8100 + world)
    from w4_gemm_error_b200 import spear
    for M in (1, 9, 40):
        x = make_x(M, 1032, seed=100 * world + M)
        g.check(x, g.call(x), what=f"world {world} M={M}")
        g.check(x, g.call(x, spear.SPEAR_EC_OFF), ec_on=False, what=f"world {world} M={M} EC off")
    assert g.status() == [0] * world
    g.close()


def test_layer_without_ec():
    g = Group(512, 264, 0, 2, 16, seed=8200)
    for M in (3, 16):
        x = make_x(M, 512, seed=M)
        g.check(x, g.call(x), what=f"r=0 M={M}")
    g.close()


def test_prefill_sized_shards():
    """300 tokens: the shards' forward takes the dispatch table's larger-batch
    path, and the push form of the prepass splits K over CTAs with several
    token tiles."""
    g = Group(2048, 1024, 64, 2, 300, seed=8300)
    x = make_x(300, 2048, seed=5)
    g.check(x, g.call(x), what="M=300")
    assert g.status() == [0, 0]
    g.close()


def test_repeated_calls_and_graph_replay():
    """The counts that order the ranks live on the device: eager calls and a
    CUDA graph of one call (all ranks' phases) replayed with new inputs."""
    g = Group(1024, 512, 16, 2, 8, seed=8400)
    M = 8
    for i in range(3):
        x = make_x(M, 1024, seed=40 + i)
        g.check(x, g.call(x), what=f"eager call {i}")
    xs = [torch.empty((M, k1 - k0), dtype=torch.bfloat16, device="cuda") for k0, k1 in g.bounds]
    ys = [torch.empty((M, 512), dtype=torch.bfloat16, device="cuda") for _ in g.tps]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            for t, x_p in zip(g.tps, xs):
                t.partial(x_p, 0, stream=s)
            for t, y in zip(g.tps, ys):
                t.reduce(M, 0, out=y, stream=s)
    torch.cuda.synchronize()
    for i in range(3):
        x = make_x(M, 1024, seed=50 + i)
        for buf, src in zip(xs, g.xs(x)):
            buf.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        g.check(x, [y.clone() for y in ys], what=f"graph replay {i}")
    del graph
    x = make_x(M, 1024, seed=60)
    g.check(x, g.call(x), what="eager after the graph")
    assert g.status() == [0, 0]
    g.close()


def test_connect_checks_and_call_order():
    from w4_gemm_error_b200 import spear
    from w4_gemm_error_b200.spear import W4ECRowParallel
    g = Group(512, 256, 8, 2, 4, seed=8500)
    t0, t1 = g.tps
    # entries out of rank order: the control blocks do not match
    with pytest.raises(spear.SpearError) as ei:
        t0.connect([t0.base, t0.base])
    assert ei.value.status == spear.SPEAR_ERR_INVALID
    with pytest.raises(spear.SpearError) as ei:
        t1.connect([t1.base, t0.base])     # own entry not at its rank
    assert ei.value.status == spear.SPEAR_ERR_INVALID
    x = make_x(2, 512, seed=1)
    with pytest.raises(spear.SpearError) as ei:
        t0.partial(g.xs(x)[0])             # the failed connects left t0 unconnected
    assert ei.value.status == spear.SPEAR_ERR_STATE
    # a rank of another group size
    other = W4ECRowParallel(g.shards[1], 1, 3, 4)
    with pytest.raises(spear.SpearError) as ei:
        t0.connect([t0.base, other.base])
    assert ei.value.status == spear.SPEAR_ERR_INVALID
    other.close()
    with pytest.raises(spear.SpearError) as ei:
        W4ECRowParallel(g.shards[0], 0, 2, 5)   # max_M above the shard's
    assert ei.value.status == spear.SPEAR_ERR_INVALID
    bases = [t.base for t in g.tps]
    for t in g.tps:
        t.connect(bases)
    with pytest.raises(spear.SpearError) as ei:
        t0.partial(make_x(5, 512, seed=2)[:, :256].contiguous().cuda())   # M above max_M
    assert ei.value.status == spear.SPEAR_ERR_INVALID
    g.check(x, g.call(x), what="after reconnecting")
    g.close()


def test_missing_rank_times_out():
    """Rank 1 never runs its partial phase: rank 0's reduce gives up after its
    bounded wait (about a second), the shard reports SPEAR_ERR_TIMEOUT, and
    the device stays usable."""
    from w4_gemm_error_b200 import spear
    g = Group(512, 256, 8, 2, 4, seed=8600)
    x = make_x(2, 512, seed=3)
    x0 = g.xs(x)[0]
    g.tps[0].partial(x0)
    g.tps[0].reduce(2)
    torch.cuda.synchronize()
    assert g.shards[0].status() == spear.SPEAR_ERR_TIMEOUT
    g.close()
    t = torch.ones(4, device="cuda")
    assert float((t * 2).sum()) == 8.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_rank(rank, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2")
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        from w4_gemm_error_b200 import spear
        from w4_gemm_error_b200.spear import W4ECLinear, W4ECRowParallel, tp_shard, tp_shard_bounds
        lay = make_layer(512, 256, 8, seed=8700)
        codes, s, z = oracle.pack(lay.W)
        k0, k1 = tp_shard_bounds(512, 2)[rank]
        c_p, s_p, z_p, A_p, wg_p = tp_shard(torch.from_numpy(codes.view(np.int32)), torch.from_numpy(s),
                                            torch.from_numpy(z), lay.A, lay.wg, k0, k1)
        lin = W4ECLinear(None, A_p.cuda(), lay.B.cuda(), wg_p.cuda(), lay.b_g, max_M=4,
                         packed=(c_p.cuda(), s_p.cuda(), z_p.cuda()))
        tp = W4ECRowParallel(lin, rank, 2, 4)
        tp.connect_group()                   # opens the other process's buffer and checks its control block
        ok = True
        try:                                 # a handle list in the wrong order is refused
            h = spear.tp_gather_handles(tp.ipc_handle(), 2)
            tp.connect_ipc(h[::-1])
            ok = False
        except spear.SpearError as e:
            ok = e.status == spear.SPEAR_ERR_INVALID
        dist.barrier()
        tp.close()
        lin.close()
        q.put((rank, ok))
    except BaseException as exc:
        q.put((rank, repr(exc)))
        raise
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_ipc_handles_connect_two_processes():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, True), (1, True)]
