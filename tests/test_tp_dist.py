"""Host side of the tensor-parallel layer on CPU: the shard bounds, the shard
slicing of the binding (split along K, and along N for column parallelism),
the handle exchange over a process group, and the row-parallel
decomposition the library's kernels implement, checked with two and three
gloo ranks against the fp64 oracle of the whole layer.

The decomposition (SPEAR, Abstract: the input-dependent gate is what makes
tensor-parallel ranks synchronise): with rank p holding the input features
[k0_p, k1_p),
    y = sum_p x_p.W^_p^T + sigmoid(sum_p x_p.w_g,p + b_g) . ((sum_p x_p.A_p) . B),
every rank's partial output being the oracle's plain W4 product of its
shard (the whole rows' scales), and its EC partial x_p.[w_g,p, A_p].
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_bounds_cover_k_in_whole_words():
    from w4_gemm_error_b200.spear import tp_shard_bounds
    for K in (8, 64, 776, 1032, 4096, 14336):
        for world in range(1, 9):
            if K // 8 < world:
                with pytest.raises(ValueError):
                    tp_shard_bounds(K, world)
                continue
            b = tp_shard_bounds(K, world)
            assert len(b) == world and b[0][0] == 0 and b[-1][1] == K
            for (k0, k1), (n0, _) in zip(b, b[1:]):
                assert k1 == n0
            sizes = [k1 - k0 for k0, k1 in b]
            assert all(s > 0 and s % 8 == 0 for s in sizes)
            assert max(sizes) - min(sizes) <= 8
    for K, world in ((12, 1), (64, 0), (64, 9)):
        with pytest.raises(ValueError):
            tp_shard_bounds(K, world)


def test_shard_slices_the_exported_layout():
    """codes[:, k0/8:k1/8] holds exactly the codes of features k0..k1-1 (the
    exported layout puts k = 8j + i in bits 4i..4i+3 of word j)."""
    from w4_gemm_error_b200.spear import tp_shard
    rng = np.random.default_rng(0)
    N, K = 5, 64
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint32)
    codes = np.zeros((N, K // 8), dtype=np.uint32)
    for i in range(8):
        codes |= q[:, i::8] << (4 * i)
    A = rng.standard_normal((K, 3))
    wg = rng.standard_normal(K)
    s = np.ones(N, dtype=np.float32)
    z = np.full(N, 8, dtype=np.uint8)
    part, s2, z2, A2, wg2 = tp_shard(codes, s, z, A, wg, 16, 40)
    assert part.shape == (N, 3) and part.flags.c_contiguous
    back = np.stack([(part >> (4 * i)) & 15 for i in range(8)], axis=-1).reshape(N, 24)
    assert np.array_equal(back, q[:, 16:40])
    assert np.array_equal(A2, A[16:40]) and np.array_equal(wg2, wg[16:40])
    assert s2 is s and z2 is z
    with pytest.raises(ValueError):
        tp_shard(codes, s, z, A, wg, 4, 40)


def _f64(t):
    return t.float().double().numpy()


@pytest.mark.parametrize("world", [2, 3])
def test_column_shards_give_the_columns_of_the_whole_layer(world):
    """Split along N, each rank's oracle forward is exactly its columns of
    the whole layer's (same u and gate on every rank, same sums per
    element), with the EC on and off."""
    import oracle
    from w4_gemm_error_b200.inputs import make_layer, make_x
    from w4_gemm_error_b200.spear import tp_column_shard, tp_shard_bounds
    M, K, N, r = 3, 264, 200, 12
    lay = make_layer(K, N, r, seed=21)
    x = make_x(M, K, seed=21)
    codes, s, z = oracle.pack(lay.W)
    for ec_on in (True, False):
        ref = oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g, ec_on=ec_on)
        cols = []
        for n0, n1 in tp_shard_bounds(N, world):
            c_p, s_p, z_p, B_p = tp_column_shard(codes, s, z, lay.B, n0, n1)
            assert c_p.shape == (n1 - n0, K // 8) and B_p.shape == (r, n1 - n0)
            cols.append(oracle.forward(x, c_p, s_p, z_p, lay.A, B_p, lay.wg, lay.b_g, ec_on=ec_on))
        assert np.array_equal(np.concatenate(cols, axis=1), ref)
    with pytest.raises(ValueError):
        tp_column_shard(codes, s, z, lay.B, 4, 16)


def _rank_main(rank, world, port, q, case):
    import datetime
    import sys
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import oracle
        from w4_gemm_error_b200.inputs import make_layer, make_x
        from w4_gemm_error_b200.spear import tp_gather_handles, tp_shard, tp_shard_bounds
        M, K, N, r, seed = case
        lay = make_layer(K, N, r, seed=seed)          # every rank draws the same layer and input
        x = make_x(M, K, seed=seed)
        codes, s, z = oracle.pack(lay.W)
        k0, k1 = tp_shard_bounds(K, world)[rank]
        c_p, s_p, z_p, A_p, wg_p = tp_shard(codes, s, z, lay.A, lay.wg, k0, k1)
        x_p = x[:, k0:k1].contiguous()
        y_p = oracle.forward(x_p, c_p, s_p, z_p, A_p, lay.B, wg_p, lay.b_g, ec_on=False)
        if r:
            G_p = np.concatenate([_f64(wg_p)[:, None], _f64(A_p)], axis=1)   # [k, r + 1]
            u_p = _f64(x_p) @ G_p
        else:
            u_p = np.zeros((M, 1))
        # the exchange: every rank's partials in rank order
        parts = [None] * world
        dist.all_gather_object(parts, (rank, y_p, u_p))
        handles = tp_gather_handles(bytes([rank]) * 64, world)
        assert [h[0] for h in handles] == list(range(world))
        try:   # one rank with a short handle: every rank refuses the gathered list
            tp_gather_handles(b"x" * (63 if rank == world - 1 else 64), world)
            raise AssertionError("a short handle was accepted")
        except ValueError:
            pass
        assert [p[0] for p in parts] == list(range(world))
        y = sum(p[1] for p in parts)
        if r:
            u = sum(p[2] for p in parts)
            g = 1.0 / (1.0 + np.exp(-(u[:, 0] + lay.b_g)))
            y = y + g[:, None] * (u[:, 1:] @ _f64(lay.B))
        ref = oracle.forward(x, codes, s, z, lay.A, lay.B, lay.wg, lay.b_g)
        err = float(np.max(np.abs(y - ref) / (1e-12 + np.abs(ref).max())))
        q.put((rank, err, (k0, k1)))
    except BaseException as exc:   # report at once instead of letting the parent wait
        q.put((rank, repr(exc), None))
        raise
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [(2, (5, 1032, 264, 20, 11)), (3, (3, 776, 200, 33, 12)),
                                        (2, (4, 512, 136, 0, 13))])
def test_ranks_reassemble_the_whole_layer(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, case)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == list(range(world))
    for rank, err, bounds in out:
        assert bounds is not None, (rank, err)
    assert out[0][2][0] == 0 and out[-1][2][1] == case[1]
    for rank, err, _ in out:
        assert err < 1e-12, (rank, err)


def _connect_rank(rank, world, port, q):
    """connect_group of the binding over gloo, with the two library calls it
    makes replaced by recorders (no GPU here)."""
    import datetime
    import sys
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        from w4_gemm_error_b200 import spear
        seen = {}
        spear.spear_w4ec_tp_ipc_handle = lambda h: bytes([10 + rank]) * spear.SPEAR_TP_IPC_HANDLE_BYTES
        spear.spear_w4ec_tp_connect_ipc = lambda h, handles: seen.setdefault("handles", list(handles))
        tp = object.__new__(spear.W4ECRowParallel)   # no device: only the host logic runs
        tp.h, tp.rank, tp.world = 1234, rank, world
        tp.connect_group()
        tp.h = None                                    # nothing to destroy
        q.put((rank, [h[0] for h in seen["handles"]]))
    except BaseException as exc:
        q.put((rank, repr(exc)))
        raise
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_connect_group_hands_every_rank_the_handles_in_rank_order(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_connect_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [10 + r for r in range(world)]
    assert out == [(r, want) for r in range(world)]
