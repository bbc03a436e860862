"""Python binding of libspear_w4ec (ctypes): argument marshalling only.

Every function here has the name of the C entry point it calls
(include/spear_w4ec.h) and does no arithmetic of its own: PyTorch provides
device memory and streams, the library's kernels do all the work.  If the
shared library is missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspear_w4ec.so")

SPEAR_OK = 0
SPEAR_ERR_INVALID = -1
SPEAR_ERR_UNSUPPORTED = -2
SPEAR_ERR_NOMEM = -3
SPEAR_ERR_CUDA = -4
SPEAR_ERR_TIMEOUT = -5
SPEAR_ERR_DEVICE = -6
SPEAR_ERR_STATE = -7

SPEAR_EC_OFF = 1
SPEAR_FORCE_FUSED = 2
SPEAR_FORCE_SPLIT = 4
SPEAR_FORCE_DECODE = 8
SPEAR_FORCE_TC = 16
SPEAR_STACK_PERSISTENT = 32   # stack forward only: one persistent kernel for the whole stack

SPEAR_TP_MAX_WORLD = 8
SPEAR_TP_IPC_HANDLE_BYTES = 64

EXPORTED = ("spear_w4ec_create", "spear_w4ec_pack", "spear_w4ec_pack_asym", "spear_w4ec_import",
            "spear_w4ec_forward", "spear_w4ec_forward_host",
            "spear_w4ec_destroy", "spear_w4ec_get_packed", "spear_w4ec_get_gate", "spear_w4ec_sync_status",
            "spear_w4ec_tune", "spear_w4ec_dispatch", "spear_w4ec_gate_noalloc", "spear_w4ec_set_next",
            "spear_w4ec_stack_create", "spear_w4ec_stack_forward", "spear_w4ec_stack_forward_host",
            "spear_w4ec_stack_buffer", "spear_w4ec_stack_destroy", "spear_w4ec_cost", "spear_w4ec_table_save",
            "spear_w4ec_table_load", "spear_w4ec_tp_create", "spear_w4ec_tp_buffer", "spear_w4ec_tp_ipc_handle",
            "spear_w4ec_tp_connect_ipc", "spear_w4ec_tp_connect", "spear_w4ec_tp_partial", "spear_w4ec_tp_reduce",
            "spear_w4ec_tp_forward", "spear_w4ec_tp_destroy", "spear_w4ec_strerror")


class SpearError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {strerror(status)} ({status})")


class _Opts(ctypes.Structure):
    _fields_ = [("max_M", ctypes.c_int64), ("device", ctypes.c_int32)]


class StackOp(ctypes.Structure):
    """spear_w4ec_stack_op: the layer handle, the buffers it reads and writes,
    and whether its EC is placed (1) or not (0)."""
    _fields_ = [("layer", ctypes.c_void_p), ("in_", ctypes.c_int32), ("out", ctypes.c_int32),
                ("ec", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m w4_gemm_error_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, u32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_float
    sig = {
        "spear_w4ec_create": [ctypes.POINTER(P), i64, i64, i32, ctypes.POINTER(_Opts)],
        "spear_w4ec_pack": [P, P, P, P, P, f32, P],
        "spear_w4ec_pack_asym": [P, P, P, P, P, f32, P],
        "spear_w4ec_import": [P, P, P, P, P, P, P, f32, P],
        "spear_w4ec_forward": [P, P, P, i64, u32, P],
        "spear_w4ec_forward_host": [P, P, P, i64, u32, P],
        "spear_w4ec_destroy": [P],
        "spear_w4ec_get_packed": [P, P, P, P, P],
        "spear_w4ec_get_gate": [P, P, P, i64, P],
        "spear_w4ec_sync_status": [P, P],
        "spear_w4ec_tune": [P, P, P, i64, P, ctypes.POINTER(u32)],
        "spear_w4ec_dispatch": [P, i64, ctypes.POINTER(u32)],
        "spear_w4ec_gate_noalloc": [P, i64, i64, P, f32, P, P],
        "spear_w4ec_set_next": [P, P],
        "spear_w4ec_stack_create": [ctypes.POINTER(P), ctypes.POINTER(StackOp), i32, i64],
        "spear_w4ec_stack_forward": [P, P, P, i64, u32, P],
        "spear_w4ec_stack_forward_host": [P, P, P, i64, u32, P],
        "spear_w4ec_stack_buffer": [P, i32, ctypes.POINTER(P)],
        "spear_w4ec_stack_destroy": [P],
        "spear_w4ec_cost": [P, i64, u32, ctypes.POINTER(f32)],
        "spear_w4ec_table_save": [P, ctypes.c_char_p, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)],
        "spear_w4ec_table_load": [P, ctypes.c_char_p],
        "spear_w4ec_tp_create": [ctypes.POINTER(P), P, i32, i32, i64],
        "spear_w4ec_tp_buffer": [P, ctypes.POINTER(P), ctypes.POINTER(ctypes.c_size_t),
                                 ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)],
        "spear_w4ec_tp_ipc_handle": [P, P],
        "spear_w4ec_tp_connect_ipc": [P, P],
        "spear_w4ec_tp_connect": [P, ctypes.POINTER(P)],
        "spear_w4ec_tp_partial": [P, P, i64, u32, P],
        "spear_w4ec_tp_reduce": [P, P, i64, u32, P],
        "spear_w4ec_tp_forward": [P, P, P, i64, u32, P],
        "spear_w4ec_tp_destroy": [P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.spear_w4ec_strerror.argtypes = [ctypes.c_int]
    lib.spear_w4ec_strerror.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def strerror(status: int) -> str:
    return _lib.spear_w4ec_strerror(int(status)).decode()


def _check(rc: int, call: str):
    if rc != SPEAR_OK:
        raise SpearError(rc, call)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return ctypes.c_void_p(t.data_ptr())
    return ctypes.c_void_p(int(t))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev_bf16(t: torch.Tensor, shape, name):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and tuple(t.shape) == tuple(shape)):
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor of shape {tuple(shape)}")


def spear_w4ec_create(K: int, N: int, r: int, max_M: int = 4096, device: int = -1) -> int:
    h = ctypes.c_void_p()
    opts = _Opts(max_M, device)
    _check(_lib.spear_w4ec_create(ctypes.byref(h), K, N, r, ctypes.byref(opts)), "spear_w4ec_create")
    return h.value


def spear_w4ec_pack(h: int, W, A, B, w_g, b_g: float, stream=None):
    _check(_lib.spear_w4ec_pack(h, _ptr(W), _ptr(A), _ptr(B), _ptr(w_g), float(b_g), _stream(stream)),
           "spear_w4ec_pack")


def spear_w4ec_pack_asym(h: int, W, A, B, w_g, b_g: float, stream=None):
    _check(_lib.spear_w4ec_pack_asym(h, _ptr(W), _ptr(A), _ptr(B), _ptr(w_g), float(b_g), _stream(stream)),
           "spear_w4ec_pack_asym")


def spear_w4ec_import(h: int, codes, s, z, A, B, w_g, b_g: float, stream=None):
    _check(_lib.spear_w4ec_import(h, _ptr(codes), _ptr(s), _ptr(z), _ptr(A), _ptr(B), _ptr(w_g), float(b_g),
                                  _stream(stream)), "spear_w4ec_import")


def spear_w4ec_forward(h: int, x, y, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_forward(h, _ptr(x), _ptr(y), M, flags, _stream(stream)), "spear_w4ec_forward")


def spear_w4ec_forward_host(h: int, x_host, y_host, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_forward_host(h, _ptr(x_host), _ptr(y_host), M, flags, _stream(stream)),
           "spear_w4ec_forward_host")


def spear_w4ec_destroy(h: int):
    _check(_lib.spear_w4ec_destroy(h), "spear_w4ec_destroy")


def spear_w4ec_get_packed(h: int, codes=None, s=None, z=None, stream=None):
    _check(_lib.spear_w4ec_get_packed(h, _ptr(codes), _ptr(s), _ptr(z), _stream(stream)), "spear_w4ec_get_packed")


def spear_w4ec_get_gate(h: int, x, g, M: int, stream=None):
    _check(_lib.spear_w4ec_get_gate(h, _ptr(x), _ptr(g), M, _stream(stream)), "spear_w4ec_get_gate")


def spear_w4ec_sync_status(h: int, stream=None) -> int:
    return int(_lib.spear_w4ec_sync_status(h, _stream(stream)))


def spear_w4ec_tune(h: int, x, y, M: int, stream=None) -> int:
    choice = ctypes.c_uint32(0)
    _check(_lib.spear_w4ec_tune(h, _ptr(x), _ptr(y), M, _stream(stream), ctypes.byref(choice)), "spear_w4ec_tune")
    return choice.value


def spear_w4ec_dispatch(h: int, M: int) -> int:
    choice = ctypes.c_uint32(0)
    _check(_lib.spear_w4ec_dispatch(h, M, ctypes.byref(choice)), "spear_w4ec_dispatch")
    return choice.value


def spear_w4ec_set_next(h: int, next_h):
    _check(_lib.spear_w4ec_set_next(h, next_h), "spear_w4ec_set_next")


def spear_w4ec_gate_noalloc(x, M: int, K: int, w_g, b_g: float, g, stream=None):
    """Gate g[t] for M <= 4096 tokens with no allocation (static scratch inside the library)."""
    _check(_lib.spear_w4ec_gate_noalloc(_ptr(x), M, K, _ptr(w_g), float(b_g), _ptr(g), _stream(stream)),
           "spear_w4ec_gate_noalloc")


def spear_w4ec_cost(h: int, M: int, flags: int) -> float:
    us = ctypes.c_float(0.0)
    _check(_lib.spear_w4ec_cost(h, M, flags, ctypes.byref(us)), "spear_w4ec_cost")
    return us.value


def spear_w4ec_table_save(h: int) -> str:
    n = ctypes.c_size_t(0)
    _lib.spear_w4ec_table_save(h, None, 0, ctypes.byref(n))
    buf = ctypes.create_string_buffer(n.value + 1)
    _check(_lib.spear_w4ec_table_save(h, buf, n.value + 1, ctypes.byref(n)), "spear_w4ec_table_save")
    return buf.value.decode()


def spear_w4ec_table_load(h: int, text: str):
    _check(_lib.spear_w4ec_table_load(h, text.encode()), "spear_w4ec_table_load")


def spear_w4ec_stack_create(ops, max_M: int) -> int:
    """ops: sequence of (layer handle, in, out, ec) tuples."""
    arr = (StackOp * len(ops))(*[StackOp(h, i, o, e) for (h, i, o, e) in ops])
    s = ctypes.c_void_p()
    _check(_lib.spear_w4ec_stack_create(ctypes.byref(s), arr, len(ops), max_M), "spear_w4ec_stack_create")
    return s.value


def spear_w4ec_stack_forward(s: int, x, y, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_stack_forward(s, _ptr(x), _ptr(y), M, flags, _stream(stream)), "spear_w4ec_stack_forward")


def spear_w4ec_stack_forward_host(s: int, x_host, y_host, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_stack_forward_host(s, _ptr(x_host), _ptr(y_host), M, flags, _stream(stream)),
           "spear_w4ec_stack_forward_host")


def spear_w4ec_stack_buffer(s: int, index: int) -> int:
    p = ctypes.c_void_p()
    _check(_lib.spear_w4ec_stack_buffer(s, index, ctypes.byref(p)), "spear_w4ec_stack_buffer")
    return p.value


def spear_w4ec_stack_destroy(s: int):
    _check(_lib.spear_w4ec_stack_destroy(s), "spear_w4ec_stack_destroy")


def spear_w4ec_tp_create(shard_h: int, rank: int, world: int, max_M: int) -> int:
    out = ctypes.c_void_p()
    _check(_lib.spear_w4ec_tp_create(ctypes.byref(out), shard_h, int(rank), int(world), int(max_M)),
           "spear_w4ec_tp_create")
    return out.value


def spear_w4ec_tp_buffer(t: int):
    """(device address, bytes, u-slot offset, partial-output offset) of the exchange buffer."""
    base, nbytes, uo, yo = ctypes.c_void_p(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.spear_w4ec_tp_buffer(t, ctypes.byref(base), ctypes.byref(nbytes), ctypes.byref(uo),
                                     ctypes.byref(yo)), "spear_w4ec_tp_buffer")
    return base.value, nbytes.value, uo.value, yo.value


def spear_w4ec_tp_ipc_handle(t: int) -> bytes:
    buf = ctypes.create_string_buffer(SPEAR_TP_IPC_HANDLE_BYTES)
    _check(_lib.spear_w4ec_tp_ipc_handle(t, buf), "spear_w4ec_tp_ipc_handle")
    return buf.raw


def spear_w4ec_tp_connect_ipc(t: int, handles):
    blob = b"".join(handles)
    if any(len(h) != SPEAR_TP_IPC_HANDLE_BYTES for h in handles):
        raise ValueError(f"every handle must be {SPEAR_TP_IPC_HANDLE_BYTES} bytes")
    buf = ctypes.create_string_buffer(blob, len(blob))
    _check(_lib.spear_w4ec_tp_connect_ipc(t, buf), "spear_w4ec_tp_connect_ipc")


def spear_w4ec_tp_connect(t: int, buffers):
    arr = (ctypes.c_void_p * len(buffers))(*[int(b) for b in buffers])
    _check(_lib.spear_w4ec_tp_connect(t, arr), "spear_w4ec_tp_connect")


def spear_w4ec_tp_partial(t: int, x, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_tp_partial(t, _ptr(x), M, flags, _stream(stream)), "spear_w4ec_tp_partial")


def spear_w4ec_tp_reduce(t: int, y, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_tp_reduce(t, _ptr(y), M, flags, _stream(stream)), "spear_w4ec_tp_reduce")


def spear_w4ec_tp_forward(t: int, x, y, M: int, flags: int = 0, stream=None):
    _check(_lib.spear_w4ec_tp_forward(t, _ptr(x), _ptr(y), M, flags, _stream(stream)), "spear_w4ec_tp_forward")


def spear_w4ec_tp_destroy(t: int):
    _check(_lib.spear_w4ec_tp_destroy(t), "spear_w4ec_tp_destroy")


class W4ECLinear:
    """Owning wrapper of one packed layer (create + pack; destroy on close).

    Shapes: W [N, K], A [K, r], B [r, N], w_g [K] (bf16 CUDA tensors).
    """

    def __init__(self, W: torch.Tensor | None, A: torch.Tensor | None, B: torch.Tensor | None,
                 w_g: torch.Tensor | None, b_g: float, max_M: int = 4096, stream=None, quant: str = "sym",
                 packed=None):
        """quant: "sym" (spear_w4ec_pack) or "asym" (spear_w4ec_pack_asym);
        packed: (codes int32/uint32 [N, K/8], s float32 [N], z uint8 [N]) CUDA
        tensors of a layer quantised elsewhere (spear_w4ec_import; W is None)."""
        if packed is not None:
            codes, s_, z_ = packed
            N, K = codes.shape[0], codes.shape[1] * 8
            if not (codes.is_cuda and codes.dtype in (torch.int32, torch.uint32) and codes.is_contiguous()
                    and s_.is_cuda and s_.dtype == torch.float32 and tuple(s_.shape) == (N,)
                    and z_.is_cuda and z_.dtype == torch.uint8 and tuple(z_.shape) == (N,)):
                raise ValueError("packed must be CUDA (codes [N, K/8] int32, s [N] float32, z [N] uint8)")
            device = codes.device
        else:
            N, K = W.shape
            _dev_bf16(W, (N, K), "W")
            device = W.device
        if quant not in ("sym", "asym"):
            raise ValueError("quant must be 'sym' or 'asym'")
        r = 0 if A is None else A.shape[1]
        if r:
            _dev_bf16(A, (K, r), "A")
            _dev_bf16(B, (r, N), "B")
            _dev_bf16(w_g, (K,), "w_g")
        self.K, self.N, self.r, self.max_M = K, N, r, max_M
        self.device = device
        self.h = spear_w4ec_create(K, N, r, max_M, device.index if device.index is not None else -1)
        try:
            if packed is not None:
                spear_w4ec_import(self.h, packed[0], packed[1], packed[2], A, B, w_g, b_g, stream)
            elif quant == "asym":
                spear_w4ec_pack_asym(self.h, W, A, B, w_g, b_g, stream)
            else:
                spear_w4ec_pack(self.h, W, A, B, w_g, b_g, stream)
        except Exception:
            spear_w4ec_destroy(self.h)
            self.h = None
            raise

    def forward(self, x: torch.Tensor, flags: int = 0, out: torch.Tensor | None = None, stream=None):
        M = x.shape[0]
        _dev_bf16(x, (M, self.K), "x")
        y = out if out is not None else torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        _dev_bf16(y, (M, self.N), "y")
        spear_w4ec_forward(self.h, x, y, M, flags, stream)
        return y

    __call__ = forward

    def packed(self, stream=None):
        codes = torch.empty((self.N, self.K // 8), dtype=torch.int32, device=self.device)
        s = torch.empty(self.N, dtype=torch.float32, device=self.device)
        z = torch.empty(self.N, dtype=torch.uint8, device=self.device)
        spear_w4ec_get_packed(self.h, codes, s, z, stream)
        return codes, s, z

    def gate(self, x: torch.Tensor, stream=None):
        M = x.shape[0]
        _dev_bf16(x, (M, self.K), "x")
        g = torch.empty(M, dtype=torch.float32, device=x.device)
        spear_w4ec_get_gate(self.h, x, g, M, stream)
        return g

    def status(self, stream=None) -> int:
        return spear_w4ec_sync_status(self.h, stream)

    def tune(self, x: torch.Tensor, y: torch.Tensor, stream=None) -> int:
        return spear_w4ec_tune(self.h, x, y, x.shape[0], stream)

    def dispatch(self, M: int) -> int:
        return spear_w4ec_dispatch(self.h, M)

    def cost(self, M: int, flags: int) -> float:
        """Measured microseconds of one forward with these path / placement / EC flags (after tune)."""
        return spear_w4ec_cost(self.h, M, flags)

    def table_json(self) -> str:
        return spear_w4ec_table_save(self.h)

    def load_table(self, text: str):
        spear_w4ec_table_load(self.h, text)

    def set_next(self, other: "W4ECLinear | None"):
        """Name the layer whose forward follows this one (prefetch hint; None clears)."""
        spear_w4ec_set_next(self.h, other.h if other is not None else None)
        self._next = other   # keeps it alive while named

    def close(self):
        if getattr(self, "h", None):
            spear_w4ec_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class W4ECStack:
    """Owning wrapper of a layer stack (spear_w4ec_stack_*).

    ops: sequence of (W4ECLinear, in, out, ec): buffer 0 is the input x,
    1 the output y (last op only), 2 and up intermediates; ec = 1 places the
    layer's EC, 0 runs it as the plain W4 GEMM.  The layers must stay open
    while the stack is used.
    """

    def __init__(self, ops, max_M: int):
        self.layers = [op[0] for op in ops]
        readers = [op[0].K for op in ops if op[1] == 0]
        self.in_width = readers[0] if readers else 0   # the library rejects a stack that never reads x
        self.out_width = ops[-1][0].N
        self.max_M = max_M
        self.device = ops[0][0].device
        self.h = spear_w4ec_stack_create([(lin.h, i, o, e) for (lin, i, o, e) in ops], max_M)
        self.widths = {}
        for lin, _, o, _ in ops:
            self.widths[o] = lin.N

    def forward(self, x: torch.Tensor, flags: int = 0, out: torch.Tensor | None = None, stream=None):
        M = x.shape[0]
        _dev_bf16(x, (M, self.in_width), "x")
        y = out if out is not None else torch.empty((M, self.out_width), dtype=torch.bfloat16, device=x.device)
        _dev_bf16(y, (M, self.out_width), "y")
        spear_w4ec_stack_forward(self.h, x, y, M, flags, stream)
        return y

    __call__ = forward

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, flags: int = 0, stream=None):
        M = x_host.shape[0]
        if x_host.is_cuda or y_host.is_cuda or tuple(x_host.shape) != (M, self.in_width) or \
                tuple(y_host.shape) != (M, self.out_width) or x_host.dtype != torch.bfloat16 or \
                y_host.dtype != torch.bfloat16 or not (x_host.is_contiguous() and y_host.is_contiguous()):
            raise ValueError("x_host, y_host must be contiguous host bf16 tensors [M, in] and [M, out]")
        spear_w4ec_stack_forward_host(self.h, x_host, y_host, M, flags, stream)
        return y_host

    def buffer(self, index: int, M: int) -> torch.Tensor:
        """A copy of intermediate buffer ``index`` as written by the last forward on M tokens."""
        ptr = spear_w4ec_stack_buffer(self.h, index)
        width = self.widths[index]

        class _View:   # the buffer's first M rows, seen through the CUDA array interface
            __cuda_array_interface__ = {"shape": (M, width), "typestr": "<i2", "data": (ptr, False),
                                        "version": 2, "strides": None}

        torch.cuda.synchronize(self.device)
        return torch.as_tensor(_View(), device=self.device).view(torch.bfloat16).clone()

    def close(self):
        if getattr(self, "h", None):
            spear_w4ec_stack_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tp_shard_bounds(K: int, world: int):
    """Input-feature range [k0, k1) of every rank of a layer of K features
    split along K over ``world`` ranks: contiguous, in rank order, whole words
    of the exported code layout (multiples of 8), sizes within 8 of each other."""
    if K % 8 or not 1 <= world <= SPEAR_TP_MAX_WORLD or K // 8 < world:
        raise ValueError(f"K = {K} must be a multiple of 8 with at least 8 features per rank "
                         f"(1 <= world = {world} <= {SPEAR_TP_MAX_WORLD})")
    words = K // 8
    return [(8 * (words * p // world), 8 * (words * (p + 1) // world)) for p in range(world)]


def _contig(a):
    if isinstance(a, torch.Tensor):
        return a.contiguous()
    import numpy as np
    return np.ascontiguousarray(a)


def tp_shard(codes, s, z, A, w_g, k0: int, k1: int):
    """One rank's part of a packed layer: (codes[:, k0/8:k1/8], s, z, A[k0:k1],
    w_g[k0:k1]), the codes in the exported layout [N][K/8] and s, z those of
    the whole rows; B and b_g are whole on every rank.  Slicing only (torch
    tensors or NumPy arrays); A and w_g may be None for a layer without an EC."""
    if k0 % 8 or k1 % 8 or not 0 <= k0 < k1 <= codes.shape[1] * 8:
        raise ValueError(f"bad range [{k0}, {k1})")
    part = _contig(codes[:, k0 // 8:k1 // 8])
    return (part, s, z, None if A is None else _contig(A[k0:k1]), None if w_g is None else _contig(w_g[k0:k1]))


def tp_column_shard(codes, s, z, B, n0: int, n1: int):
    """One rank's part of a layer split along N (column parallelism: no
    exchange, each rank an ordinary handle of its output channels):
    (codes[n0:n1], s[n0:n1], z[n0:n1], B[:, n0:n1]); A, w_g and b_g are
    whole on every rank, so every rank forms the same u and gate and its
    forward gives y[:, n0:n1].  Slicing only; tp_shard_bounds(N, world)
    gives ranges of whole 8-row groups (a handle's N is a multiple of 8)."""
    if n0 % 8 or n1 % 8 or not 0 <= n0 < n1 <= codes.shape[0]:
        raise ValueError(f"bad range [{n0}, {n1})")
    return (_contig(codes[n0:n1]), _contig(s[n0:n1]), _contig(z[n0:n1]),
            None if B is None else _contig(B[:, n0:n1]))


def tp_gather_handles(handle: bytes, world: int, group=None):
    """Every rank's exchange-buffer handle, in rank order, gathered over a
    torch.distributed process group (any backend)."""
    import torch.distributed as dist
    out = [None] * world
    dist.all_gather_object(out, handle, group=group)
    if len(out) != world or any(not isinstance(h, bytes) or len(h) != SPEAR_TP_IPC_HANDLE_BYTES for h in out):
        raise ValueError("the group did not return one handle per rank")
    return out


def _device_copy(ptr: int, shape, typestr: str, dtype, device):
    class _View:   # device memory seen through the CUDA array interface
        __cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                    "version": 2, "strides": None}

    torch.cuda.synchronize(device)
    return torch.as_tensor(_View(), device=device).view(dtype).clone()


class W4ECRowParallel:
    """One rank of a layer split along K over ``world`` ranks
    (spear_w4ec_tp_*).  ``shard`` is the rank's W4ECLinear: K = k1 - k0 of
    tp_shard_bounds, made with ``packed=`` from tp_shard of the whole layer's
    packed codes; it must stay open while this object is used.  Connect once
    (connect_group over a process group, or connect with buffer addresses of
    ranks in this process), then call forward (or partial and reduce) on
    every rank with the same M and flags."""

    def __init__(self, shard: W4ECLinear, rank: int, world: int, max_M: int):
        self.shard, self.rank, self.world, self.max_M = shard, rank, world, max_M
        self.K, self.N, self.r = shard.K, shard.N, shard.r
        self.device = shard.device
        self.h = spear_w4ec_tp_create(shard.h, rank, world, max_M)
        self.base, self.nbytes, self.u_off, self.y_off = spear_w4ec_tp_buffer(self.h)
        self.R1p = (self.r + 1 + 15) // 16 * 16 if self.r else 16

    def ipc_handle(self) -> bytes:
        return spear_w4ec_tp_ipc_handle(self.h)

    def connect(self, buffers):
        spear_w4ec_tp_connect(self.h, buffers)

    def connect_ipc(self, handles):
        spear_w4ec_tp_connect_ipc(self.h, handles)

    def connect_group(self, group=None):
        self.connect_ipc(tp_gather_handles(self.ipc_handle(), self.world, group))

    def partial(self, x: torch.Tensor, flags: int = 0, stream=None):
        M = x.shape[0]
        _dev_bf16(x, (M, self.K), "x")
        spear_w4ec_tp_partial(self.h, x, M, flags, stream)

    def reduce(self, M: int, flags: int = 0, out: torch.Tensor | None = None, stream=None):
        y = out if out is not None else torch.empty((M, self.N), dtype=torch.bfloat16, device=self.device)
        _dev_bf16(y, (M, self.N), "y")
        spear_w4ec_tp_reduce(self.h, y, M, flags, stream)
        return y

    def forward(self, x: torch.Tensor, flags: int = 0, out: torch.Tensor | None = None, stream=None):
        M = x.shape[0]
        _dev_bf16(x, (M, self.K), "x")
        y = out if out is not None else torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        _dev_bf16(y, (M, self.N), "y")
        spear_w4ec_tp_forward(self.h, x, y, M, flags, stream)
        return y

    __call__ = forward

    def u_slots(self, M: int) -> torch.Tensor:
        """A copy of this rank's u slots after a call on M tokens: [world, M, R1p]
        fp32, slot q holding rank q's x_q.[w_g, A_q] (entries beyond r zero)."""
        rows = [_device_copy(self.base + self.u_off + 4 * q * self.max_M * self.R1p, (M, self.R1p), "<f4",
                             torch.float32, self.device) for q in range(self.world)]
        return torch.stack(rows)

    def partial_output(self, M: int) -> torch.Tensor:
        """A copy of this rank's partial output x_p.W^_p^T (bf16 [M, N]) after a call."""
        return _device_copy(self.base + self.y_off, (M, self.N), "<i2", torch.bfloat16, self.device)

    def close(self):
        if getattr(self, "h", None):
            spear_w4ec_tp_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
