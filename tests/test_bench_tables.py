"""Host-side checks of bench.py's tables (CPU only): every workload has a
traffic entry for each of its batch sizes in the bench's data file
(bench_traffic.json), each entry names kernel sources that exist, and the
algorithmic byte and flop counts follow their definitions."""
from __future__ import annotations

import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    import importlib
    import sys
    sys.path.insert(0, ROOT)
    return importlib.import_module("bench")


def test_every_workload_has_traffic_for_every_batch_size(bench):
    traffic = bench.load_traffic()
    for name, wl in bench.WORKLOADS.items():
        assert name in traffic, name
        t = traffic[name]
        assert sorted(t["bytes"]) == sorted(wl["Ms"]), name
        assert len(t["sha"]) == 16
        for f in t["files"]:
            assert os.path.exists(os.path.join(ROOT, "w4_gemm_error_b200", "csrc", f)), f


def test_traffic_is_close_to_the_algorithmic_bytes(bench):
    """Measured DRAM bytes per launch of the decode kernels stay within a few
    per cent of the algorithmic bytes (no re-reads); the tcgen05 kernel's may
    be lower (its output partly stays in L2)."""
    traffic = bench.load_traffic()
    for name, wl in bench.WORKLOADS.items():
        for M, measured in traffic[name]["bytes"].items():
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


def test_bf16_denominator_follows_the_timed_region(bench):
    peaks = {"bf16": 1651.4, "bf16_sustained": 1399.6, "source": "measured"}
    assert bench._timed_region_peak(peaks, 0.14)[0] == 1651.4
    assert bench._timed_region_peak(peaks, 5.0)[0] == 1399.6
