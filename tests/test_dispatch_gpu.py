"""Adaptive dispatch: the tuned table saved as JSON and loaded into another
handle, and the measured costs a scheduler reads (spear_w4ec_tune /
_table_save / _table_load / _cost).

SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
Efficient Low-Bit LLM Serving", Abstract: adaptive kernel-fusion dispatch,
and an EC-aware scheduler that needs the price of the EC per configuration.
"""
from __future__ import annotations

import json

import pytest
import torch

from helpers import Problem, assert_close

pytestmark = pytest.mark.gpu

FUSED, SPLIT, DECODE, TC, EC_OFF = 2, 4, 8, 16, 1


def test_tuned_table_round_trips_and_is_followed():
    from w4_gemm_error_b200 import spear
    P = Problem(16, 4096, 1024, 32, seed=60, max_M=64)
    Q = Problem(16, 4096, 1024, 32, seed=61, max_M=64)
    y = torch.empty((16, 1024), dtype=torch.bfloat16, device="cuda")
    choices = {}
    for M in (1, 16, 64):
        x = P.xd[:M].contiguous() if M <= 16 else torch.cat([P.xd] * 4)[:M].contiguous()
        choices[M] = P.lin.tune(x, torch.empty((M, 1024), dtype=torch.bfloat16, device="cuda"))
    text = P.lin.table_json()
    doc = json.loads(text)
    assert doc["K"] == 4096 and doc["N"] == 1024 and doc["r"] == 32 and len(doc["buckets"]) == 3
    # every tuned bucket lists the times of both paths with and without the EC
    for b in doc["buckets"]:
        assert b["choice"] in ("decode+fused", "decode+split", "tcgen05+fused", "tcgen05+split")
        for name in ("tcgen05+fused", "tcgen05+split", "tcgen05+fused+ec_off"):
            assert b["us"][name] > 0
    # the measured costs, as a scheduler reads them
    for M in (1, 16, 64):
        on = P.lin.cost(M, choices[M])
        off = P.lin.cost(M, (choices[M] & (DECODE | TC)) | FUSED | EC_OFF)
        assert on > 0 and off > 0
    with pytest.raises(spear.SpearError) as ei:
        P.lin.cost(300, TC | FUSED)                   # bucket never tuned
    assert ei.value.status == spear.SPEAR_ERR_STATE
    # loaded into a fresh handle of the same shape: the same choices, followed
    Q.lin.load_table(text)
    for M in (1, 16, 64):
        assert Q.lin.dispatch(M) == choices[M]
    assert Q.lin.table_json() == text
    y = Q.lin(Q.xd)
    torch.cuda.synchronize()
    assert Q.lin.status() == 0
    assert_close(y, Q.oracle_y(), "forward with the loaded table")
    P.close()
    Q.close()


def test_table_load_rejects_bad_text_and_other_shapes():
    from w4_gemm_error_b200 import spear
    P = Problem(4, 1024, 512, 16, seed=62)
    before = P.lin.dispatch(4)
    good = {"format": "spear_w4ec dispatch table", "version": 1, "K": 1024, "N": 512, "r": 16,
            "buckets": [{"bucket": 2, "M_max": 4, "choice": "tcgen05+split", "us": {"tcgen05+split": 9.5}}]}
    bad_texts = [
        "not json",
        json.dumps(dict(good, K=2048)),                                    # another shape
        json.dumps(dict(good, version=2)),
        json.dumps(dict(good, buckets=[{"bucket": 9, "choice": None}])),   # no such bucket
        json.dumps(dict(good, buckets=[{"bucket": 2, "choice": "decode+fused+ec_off"}])),
        json.dumps(dict(good, buckets=[{"bucket": 2, "choice": "fast"}])),
        json.dumps(dict(good, buckets=[{"bucket": 2, "choice": "tcgen05+fused", "us": {"tcgen05+fused": -1}}])),
        json.dumps(good) + " trailing",
    ]
    for text in bad_texts:
        with pytest.raises(spear.SpearError) as ei:
            P.lin.load_table(text)
        assert ei.value.status == spear.SPEAR_ERR_INVALID, text
        assert P.lin.dispatch(4) == before           # nothing changed
    P.lin.load_table(json.dumps(good))
    assert P.lin.dispatch(4) == TC | SPLIT
    assert P.lin.cost(4, TC | SPLIT) == pytest.approx(9.5)
    assert_close(P.lin(P.xd), P.oracle_y(), "loaded choice")
    P.close()
