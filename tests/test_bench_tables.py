"""Host-side checks of bench.py's tables (CPU only): every workload has a
traffic entry for each of its batch sizes, each entry names kernel sources
that exist and a committed profile summary that quotes the same source hash,
and the algorithmic byte and flop counts follow their definitions."""
from __future__ import annotations

import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    import importlib
    import sys
    sys.path.insert(0, ROOT)
    return importlib.import_module("bench")


def test_every_workload_has_traffic_for_every_batch_size(bench):
    for name, wl in bench.WORKLOADS.items():
        assert name in bench.TRAFFIC, name
        t = bench.TRAFFIC[name]
        assert sorted(t["bytes"]) == sorted(wl["Ms"]), name
        for f in t["files"]:
            assert os.path.exists(os.path.join(ROOT, "w4_gemm_error_b200", "csrc", f)), f


def test_profile_summaries_quote_the_traffic_hash(bench):
    for name, t in bench.TRAFFIC.items():
        path = os.path.join(ROOT, t["profile"])
        assert os.path.exists(path), path
        text = open(path).read()
        hashes = re.findall(r"SHA-256 prefix `([0-9a-f]{16})`", text)
        assert t["sha"] in hashes, (name, t["sha"], hashes)


def test_traffic_is_close_to_the_algorithmic_bytes(bench):
    """Measured DRAM bytes per launch of the decode kernels stay within a few
    per cent of the algorithmic bytes (no re-reads); the tcgen05 kernel's may
    be lower (its output partly stays in L2)."""
    for name, wl in bench.WORKLOADS.items():
        t = bench.TRAFFIC[name]
        for M, measured in t["bytes"].items():
            alg = bench.alg_bytes(M, wl["K"], wl["N"], wl["r"])
            assert measured <= 1.15 * alg, (name, M, measured, alg)
            if wl["kind"] == "decode" and M <= 16:
                assert measured >= 0.98 * alg, (name, M, measured, alg)


def test_algorithmic_counts(bench):
    # one q/o forward at one token: codes N*K/2, s (4 B) and z (1 B) per row,
    # A and w_g (K x (r + 1) bf16), B (r x N bf16), x and y
    K = N = 4096
    r = 32
    assert bench.alg_bytes(1, K, N, r) == N * K // 2 + 5 * N + 2 * K * (r + 1) + 2 * r * N + 2 * K + 2 * N
    assert bench.alg_flops(1, K, N, r) == 2 * N * K + 2 * K + 2 * K * r + 2 * r * N
    assert bench.packed_bytes(K, N, r) == N * K // 2 + 5 * N + 2 * K * (r + 1) + 2 * r * N
