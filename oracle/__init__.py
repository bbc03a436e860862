"""fp64 CPU oracle of the W4 + gated-EC linear layer (ctypes over oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg are the only callers.  The CUDA
library never imports or links this package, and this package imports
nothing from the CUDA library.

Functions take and return NumPy arrays; bf16 tensors are passed as their raw
uint16 bit patterns.  See oracle.c for the definition each one follows
(SPEAR, Abstract, for what the layer is; the equations are this library's
reading, restated at the top of oracle.c).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off", "-std=c11"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc), if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Lib:
    """ctypes view of one compiled copy of oracle.c."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        lib.oracle_pack.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_pack_asym.argtypes = [P, i64, i64, P, P, P]
        lib.oracle_gate.argtypes = [P, i64, i64, P, f64, P]
        lib.oracle_forward.argtypes = [P, i64, i64, i64, i32, P, P, P, P, P, P, f64, i32, P, P, P]
        lib.oracle_forward_sampled.argtypes = [P, i64, i64, i64, i32, P, P, P, P, P, P, f64, i32,
                                               P, P, i64, P]
        lib.oracle_num_threads.argtypes = []
        for f in (lib.oracle_pack, lib.oracle_pack_asym, lib.oracle_gate, lib.oracle_forward,
                  lib.oracle_forward_sampled, lib.oracle_num_threads):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = path


def load_from(path: str) -> "_Lib":
    """Load another compiled copy of oracle.c (the tests use this for mutants)."""
    return _Lib(path)


def _load() -> "_Lib":
    global _lib
    with _lock:
        if _lib is None:
            _lib = _Lib(build())
    return _lib


def _u16(a) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 array; return contiguous uint16 bits."""
    if hasattr(a, "view") and hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 operands must be torch.bfloat16 tensors or uint16 bit arrays")
    return a


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None and a.size else ctypes.c_void_p(0)


def num_threads(lib=None) -> int:
    return int((lib or _load()).lib.oracle_num_threads())


def pack(W, lib=None):
    """W bf16 [N, K] -> (codes uint32 [N, K/8], s float32 [N], z uint8 [N])."""
    W = _u16(W)
    N, K = W.shape
    codes = np.zeros((N, K // 8), dtype=np.uint32)
    s = np.zeros(N, dtype=np.float32)
    z = np.zeros(N, dtype=np.uint8)
    rc = (lib or _load()).lib.oracle_pack(_ptr(W), N, K, _ptr(codes), _ptr(s), _ptr(z))
    if rc != 0:
        raise ValueError(f"oracle_pack failed ({rc}); K must be a multiple of 8")
    return codes, s, z


def pack_asym(W, lib=None):
    """Asymmetric (min-max, stored zero point) per-channel int4 of W bf16 [N, K]
    -> (codes uint32 [N, K/8], s float32 [N], z uint8 [N])."""
    W = _u16(W)
    N, K = W.shape
    codes = np.zeros((N, K // 8), dtype=np.uint32)
    s = np.zeros(N, dtype=np.float32)
    z = np.zeros(N, dtype=np.uint8)
    rc = (lib or _load()).lib.oracle_pack_asym(_ptr(W), N, K, _ptr(codes), _ptr(s), _ptr(z))
    if rc != 0:
        raise ValueError(f"oracle_pack_asym failed ({rc}); K must be a multiple of 8")
    return codes, s, z


def gate(x, wg, b_g: float, lib=None) -> np.ndarray:
    x, wg = _u16(x), _u16(wg)
    M, K = x.shape
    g = np.zeros(M, dtype=np.float64)
    rc = (lib or _load()).lib.oracle_gate(_ptr(x), M, K, _ptr(wg), float(b_g), _ptr(g))
    if rc != 0:
        raise ValueError("oracle_gate failed")
    return g


def forward(x, codes, s, z, A, B, wg, b_g: float, *, ec_on: bool = True, want_corr: bool = False,
            lib=None):
    """y fp64 [M, N] (and g [M], corr [M, N] if ``want_corr``)."""
    x, A, B, wg = _u16(x), _u16(A), _u16(B), _u16(wg)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    z = np.ascontiguousarray(z, dtype=np.uint8)
    M, K = x.shape
    N = codes.shape[0]
    r = A.shape[1] if A.ndim == 2 else 0
    y = np.zeros((M, N), dtype=np.float64)
    g = np.zeros(M, dtype=np.float64)
    corr = np.zeros((M, N), dtype=np.float64) if want_corr else None
    rc = (lib or _load()).lib.oracle_forward(_ptr(x), M, K, N, r, _ptr(codes), _ptr(s), _ptr(z), _ptr(A), _ptr(B),
                                _ptr(wg), float(b_g), int(bool(ec_on)), _ptr(y), _ptr(g), _ptr(corr))
    if rc != 0:
        raise ValueError(f"oracle_forward failed ({rc})")
    return (y, g, corr) if want_corr else y


def forward_sampled(x, codes, s, z, A, B, wg, b_g: float, t_idx, n_idx, *, ec_on: bool = True,
                    lib=None):
    """y fp64 at the outputs (t_idx[i], n_idx[i]) only."""
    x, A, B, wg = _u16(x), _u16(A), _u16(B), _u16(wg)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    z = np.ascontiguousarray(z, dtype=np.uint8)
    t_idx = np.ascontiguousarray(t_idx, dtype=np.int64)
    n_idx = np.ascontiguousarray(n_idx, dtype=np.int64)
    M, K = x.shape
    N = codes.shape[0]
    r = A.shape[1] if A.ndim == 2 else 0
    out = np.zeros(t_idx.shape[0], dtype=np.float64)
    rc = (lib or _load()).lib.oracle_forward_sampled(_ptr(x), M, K, N, r, _ptr(codes), _ptr(s), _ptr(z), _ptr(A),
                                        _ptr(B), _ptr(wg), float(b_g), int(bool(ec_on)),
                                        _ptr(t_idx), _ptr(n_idx), t_idx.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_forward_sampled failed ({rc})")
    return out
