"""The C-ABI library loads and exports every entry point its header declares
(CPU only: no compute call needs a GPU here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"\b(spear_w4ec_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from w4_gemm_error_b200 import build
    path = build.build(quiet=True)
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("spear_w4ec_create", "spear_w4ec_pack", "spear_w4ec_forward", "spear_w4ec_destroy"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_header(lib):
    from w4_gemm_error_b200 import spear
    assert sorted(spear.EXPORTED) == _declared()
    for n in spear.EXPORTED:
        if n != "spear_w4ec_strerror":
            assert callable(getattr(spear, n))


def test_strerror_covers_every_status(lib):
    from w4_gemm_error_b200 import spear
    for st in range(0, -8, -1):
        assert spear.strerror(st) not in ("", "unknown status")
    assert spear.strerror(-99) == "unknown status"


def test_create_rejects_bad_shapes_before_touching_the_device(lib):
    from w4_gemm_error_b200 import spear
    for K, N, r in ((0, 8, 0), (12, 8, 0), (8, 12, 0), (8, 8, -1), (8, 8, 129)):
        with pytest.raises(spear.SpearError) as ei:
            spear.spear_w4ec_create(K, N, r)
        assert ei.value.status == spear.SPEAR_ERR_INVALID


def test_calls_on_null_handle_are_rejected(lib):
    from w4_gemm_error_b200 import spear
    assert spear.lib().spear_w4ec_forward(None, None, None, 1, 0, None) == spear.SPEAR_ERR_INVALID
    assert spear.lib().spear_w4ec_destroy(None) == spear.SPEAR_OK
    assert spear.lib().spear_w4ec_sync_status(None, None) == spear.SPEAR_ERR_INVALID
    assert spear.lib().spear_w4ec_set_next(None, None) == spear.SPEAR_ERR_INVALID
    assert spear.lib().spear_w4ec_dispatch(None, 1, None) == spear.SPEAR_ERR_INVALID


def test_stack_calls_reject_bad_arguments_before_touching_the_device(lib):
    from w4_gemm_error_b200 import spear
    L = spear.lib()
    s = ctypes.c_void_p()
    assert L.spear_w4ec_stack_create(None, None, 1, 1) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_stack_create(ctypes.byref(s), None, 1, 1) == spear.SPEAR_ERR_INVALID
    ops = (spear.StackOp * 1)(spear.StackOp(None, 0, 1, 1))
    assert L.spear_w4ec_stack_create(ctypes.byref(s), ops, 0, 1) == spear.SPEAR_ERR_INVALID   # no op
    assert L.spear_w4ec_stack_create(ctypes.byref(s), ops, 1, 0) == spear.SPEAR_ERR_INVALID   # max_M < 1
    assert L.spear_w4ec_stack_create(ctypes.byref(s), ops, 1, 4) == spear.SPEAR_ERR_INVALID   # NULL layer
    assert s.value is None
    assert L.spear_w4ec_stack_forward(None, None, None, 1, 0, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_stack_forward_host(None, None, None, 1, 0, None) == spear.SPEAR_ERR_INVALID
    p = ctypes.c_void_p()
    assert L.spear_w4ec_stack_buffer(None, 2, ctypes.byref(p)) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_stack_destroy(None) == spear.SPEAR_OK


def test_table_and_cost_calls_reject_bad_arguments_before_touching_the_device(lib):
    from w4_gemm_error_b200 import spear
    L = spear.lib()
    n = ctypes.c_size_t(7)
    us = ctypes.c_float(0)
    assert L.spear_w4ec_table_save(None, None, 0, ctypes.byref(n)) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_table_load(None, b"{}") == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_cost(None, 1, spear.SPEAR_FORCE_DECODE | spear.SPEAR_FORCE_FUSED, ctypes.byref(us)) \
        == spear.SPEAR_ERR_INVALID


def test_tp_calls_reject_bad_arguments_before_touching_the_device(lib):
    from w4_gemm_error_b200 import spear
    L = spear.lib()
    t = ctypes.c_void_p()
    assert L.spear_w4ec_tp_create(None, None, 0, 1, 1) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_create(ctypes.byref(t), None, 0, 1, 1) == spear.SPEAR_ERR_INVALID   # NULL shard
    assert t.value is None
    assert L.spear_w4ec_tp_buffer(None, None, None, None, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_ipc_handle(None, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_connect_ipc(None, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_connect(None, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_partial(None, None, 1, 0, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_reduce(None, None, 1, 0, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_forward(None, None, None, 1, 0, None) == spear.SPEAR_ERR_INVALID
    assert L.spear_w4ec_tp_destroy(None) == spear.SPEAR_OK
