"""ctypes binding of ``libbitnet_i2s.so`` (C ABI in ``include/bitnet_i2s.h``).

Argument marshalling only: each function takes torch CUDA tensors, checks
their dtype, device and layout, allocates outputs the caller did not pass,
and calls the C entry point of the same name on the current torch stream.
All computation happens in the library's sm_100a kernels; there is no CPU or
PyTorch fallback.  Importing this module raises if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB

BITNET_OK = 0
STATUS_NAMES = {
    0: "BITNET_OK",
    1: "BITNET_ERR_INVALID_ARG",
    2: "BITNET_ERR_SHAPE",
    3: "BITNET_ERR_ALIGN",
    4: "BITNET_ERR_CUDA",
    5: "BITNET_ERR_DEVICE_TIMEOUT",
    6: "BITNET_ERR_UNSUPPORTED",
}

# Every function the header declares, with its ctypes signature.
_I64, _VP, _SZ, _I32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "bitnet_i2s_packed_bytes": (_SZ, [_I64, _I64]),
    "bitnet_i2s_pack": (_I32, [_VP, _I64, _I64, _VP, _VP]),
    "bitnet_act_quant_i8": (_I32, [_VP, _I64, _I64, _VP, _VP, _VP]),
    "bitnet_i2s_gemv": (_I32, [_VP, _I64, _I64, _VP, _VP, _I64, _VP, _VP, _VP]),
    "bitnet_i2s_gemm": (_I32, [_VP, _I64, _I64, _VP, _VP, _I64, _VP, _VP, _VP]),
    "bitnet_i2s_dequant_f32": (_I32, [_VP, _I64, _I64, _VP, _VP]),
    "bitnet_ternarize_absmean_workspace_bytes": (_SZ, []),
    "bitnet_ternarize_absmean": (_I32, [_VP, _I64, ctypes.c_double, _VP, _VP, _VP, _SZ, _VP]),
    "bitnet_i2s_quant_gemv_workspace_bytes": (_SZ, [_I64, _I64]),
    "bitnet_i2s_quant_gemv": (_I32, [_VP, _I64, _I64, _VP, _I64, _VP, _VP, _VP, _SZ, _VP]),
    "bitnet_i2s_quant_gemv_batched_workspace_bytes": (_SZ, [_VP, _I32, _I64]),
    "bitnet_i2s_quant_gemv_batched": (_I32, [_VP, _I32, _I64, _VP, _SZ, _VP]),
    "bitnet_i2s_quant_gemv_chain_workspace_bytes": (_SZ, [_VP, _VP, _I32, _I64]),
    "bitnet_i2s_quant_gemv_chain": (_I32, [_VP, _VP, _I32, _I64, _VP, _SZ, _VP]),
    "bitnet_i2s_gemv_batched_workspace_bytes": (_SZ, [_I32]),
    "bitnet_i2s_gemv_batched": (_I32, [_VP, _I32, _I64, _VP, _SZ, _VP]),
    "bitnet_i2s_quant_gemv_noalloc": (_I32, [_VP, _I64, _I64, _VP, _I64, _VP, _VP, _VP]),
    "bitnet_iq2bn_bytes": (_SZ, [_I64, _I64]),
    "bitnet_iq1bn_bytes": (_SZ, [_I64, _I64]),
    "bitnet_iq2bn_pack": (_I32, [_VP, _I64, _I64, _I32, _VP, _VP]),
    "bitnet_iq2bn_dequant_f32": (_I32, [_VP, _I64, _I64, _I32, _VP, _VP]),
    "bitnet_iq1bn_pack": (_I32, [_VP, _I64, _I64, _VP, _VP]),
    "bitnet_iq1bn_dequant_f32": (_I32, [_VP, _I64, _I64, _VP, _VP]),
    "bitnet_iq2bn_r4_gemv": (_I32, [_VP, _I64, _I64, _VP, _VP, _I64, _VP, _VP, _VP]),
    "bitnet_debug_wait_timeout": (_I32, [_I64, _VP]),
    "bitnet_device_status": (_I32, []),
    "bitnet_last_error": (ctypes.c_char_p, []),
}


class BitnetError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"CUDA library {path} is missing; build it with `python -m i2_mpgemm_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load_library()


def _check(status: int) -> None:
    if status != BITNET_OK:
        raise BitnetError(status, lib.bitnet_last_error().decode(errors="replace"))


def _run(dev: torch.device, fn, *args, stream=None) -> None:
    """Call C entry point `fn(*args, stream)` with `dev` as the current CUDA
    device, on `stream` or, by default, the current torch stream of `dev`.
    The library works on whichever device is current, so a call on tensors of
    another device must switch to theirs first."""
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        if s.device != dev:
            raise ValueError(f"stream is on {s.device}, the tensors on {dev}")
        _check(fn(*args, s.cuda_stream or None))


def _same_device(dev: torch.device, **tensors) -> None:
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, numel: int | None = None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {numel}")


def bitnet_i2s_packed_bytes(n: int, k: int) -> int:
    return int(lib.bitnet_i2s_packed_bytes(n, k))


def bitnet_i2s_pack(w: torch.Tensor, packed: torch.Tensor | None = None, stream=None):
    """fp32 W[N,K] -> uint8 I2_S tensor of bitnet_i2s_packed_bytes(N,K) bytes."""
    _need(w, "W", torch.float32)
    n, k = w.shape
    nbytes = bitnet_i2s_packed_bytes(n, k)
    if packed is None:
        packed = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=w.device)
    _need(packed, "packed", torch.uint8, nbytes)
    _same_device(w.device, packed=packed)
    _run(w.device, lib.bitnet_i2s_pack, _ptr(w), n, k, _ptr(packed), stream=stream)
    return packed


def bitnet_act_quant_i8(x: torch.Tensor, xq: torch.Tensor | None = None,
                        xs: torch.Tensor | None = None, stream=None):
    """fp32 X[M,K] -> (int8 Xq[M,K], fp32 xs[M])."""
    _need(x, "X", torch.float32)
    m, k = x.shape
    xq = torch.empty((m, k), dtype=torch.int8, device=x.device) if xq is None else xq
    xs = torch.empty(m, dtype=torch.float32, device=x.device) if xs is None else xs
    _need(xq, "Xq", torch.int8, m * k)
    _need(xs, "xs", torch.float32, m)
    _same_device(x.device, Xq=xq, xs=xs)
    _run(x.device, lib.bitnet_act_quant_i8, _ptr(x), m, k, _ptr(xq), _ptr(xs), stream=stream)
    return xq, xs


def _matmul(fn, packed, n, k, xq, xs, y, acc, want_acc, stream):
    _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
    _need(xq, "Xq", torch.int8)
    m = xq.shape[0]
    _need(xq, "Xq", torch.int8, m * k)
    _need(xs, "xs", torch.float32, m)
    dev = packed.device
    y = torch.empty((m, n), dtype=torch.float32, device=dev) if y is None else y
    _need(y, "Y", torch.float32, m * n)
    if want_acc and acc is None:
        acc = torch.empty((m, n), dtype=torch.int32, device=dev)
    if acc is not None:
        _need(acc, "acc", torch.int32, m * n)
    _same_device(dev, Xq=xq, xs=xs, Y=y, acc=acc)
    _run(dev, fn, _ptr(packed), n, k, _ptr(xq), _ptr(xs), m, _ptr(y), _ptr(acc), stream=stream)
    return (y, acc) if acc is not None else y


def bitnet_i2s_gemv(packed, n, k, xq, xs, y=None, acc=None, want_acc=False, stream=None):
    """Decode matmul (M = Xq.shape[0] in 1..64): Y, or (Y, acc) with want_acc."""
    return _matmul(lib.bitnet_i2s_gemv, packed, n, k, xq, xs, y, acc, want_acc, stream)


def bitnet_i2s_gemm(packed, n, k, xq, xs, y=None, acc=None, want_acc=False, stream=None):
    """Matmul for any M >= 1: Y, or (Y, acc) with want_acc."""
    return _matmul(lib.bitnet_i2s_gemm, packed, n, k, xq, xs, y, acc, want_acc, stream)


def bitnet_i2s_dequant_f32(packed, n, k, w_out=None, stream=None):
    """I2_S tensor -> fp32 W[N,K] = (code - 1) * scale."""
    _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
    w_out = torch.empty((n, k), dtype=torch.float32, device=packed.device) if w_out is None else w_out
    _need(w_out, "W_out", torch.float32, n * k)
    _same_device(packed.device, W_out=w_out)
    _run(packed.device, lib.bitnet_i2s_dequant_f32, _ptr(packed), n, k, _ptr(w_out), stream=stream)
    return w_out


def bitnet_ternarize_absmean(w, eps: float = 1e-5, w_out=None, stream=None):
    """AbsMean RoundClip ternarization: (W~ * gamma as fp32, gamma as a 1-element fp64 tensor)."""
    _need(w, "W", torch.float32)
    w_out = torch.empty_like(w) if w_out is None else w_out
    _need(w_out, "W_out", torch.float32, w.numel())
    gamma = torch.empty(1, dtype=torch.float64, device=w.device)
    ws = torch.empty(int(lib.bitnet_ternarize_absmean_workspace_bytes()), dtype=torch.uint8,
                     device=w.device)
    _same_device(w.device, W_out=w_out)
    _run(w.device, lib.bitnet_ternarize_absmean, _ptr(w), w.numel(), float(eps), _ptr(w_out),
         _ptr(gamma), _ptr(ws), ws.numel(), stream=stream)
    return w_out, gamma


def bitnet_i2s_quant_gemv_workspace_bytes(m: int, k: int) -> int:
    return int(lib.bitnet_i2s_quant_gemv_workspace_bytes(m, k))


def bitnet_i2s_gemv_batched_workspace_bytes(count: int) -> int:
    return int(lib.bitnet_i2s_gemv_batched_workspace_bytes(count))


def bitnet_i2s_quant_gemv(packed, n, k, x, y=None, acc=None, workspace=None, want_acc=False,
                          stream=None):
    """Per-token quantization of fp32 X[M,K] then the matmul: Y or (Y, acc)."""
    _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
    _need(x, "X", torch.float32)
    m = x.shape[0]
    _need(x, "X", torch.float32, m * k)
    dev = packed.device
    wsb = bitnet_i2s_quant_gemv_workspace_bytes(m, k)
    if workspace is None:
        workspace = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8)
    y = torch.empty((m, n), dtype=torch.float32, device=dev) if y is None else y
    _need(y, "Y", torch.float32, m * n)
    if want_acc and acc is None:
        acc = torch.empty((m, n), dtype=torch.int32, device=dev)
    if acc is not None:
        _need(acc, "acc", torch.int32, m * n)
    _same_device(dev, X=x, Y=y, acc=acc, workspace=workspace)
    _run(dev, lib.bitnet_i2s_quant_gemv, _ptr(packed), n, k, _ptr(x), m, _ptr(y), _ptr(acc),
         _ptr(workspace), workspace.numel(), stream=stream)
    return (y, acc) if acc is not None else y


class Problem(ctypes.Structure):
    """ctypes mirror of `bitnet_i2s_problem`."""
    _fields_ = [("packed", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("X", ctypes.c_void_p), ("Y", ctypes.c_void_p), ("acc_or_null", ctypes.c_void_p)]


class BatchedQuantGemv:
    """Argument block of one bitnet_i2s_quant_gemv_batched call.

    `problems` is a list of (packed, N, K, X, Y, acc_or_None) with CUDA
    tensors; every X has M rows.  The descriptor array and the workspace are
    built once, so `run()` (capturable in a CUDA graph) only makes the call.
    """

    def __init__(self, problems, m: int, workspace: torch.Tensor | None = None):
        self.m = int(m)
        self.tensors = []  # keep every tensor alive as long as the descriptors
        arr = (Problem * len(problems))()
        for i, (packed, n, k, x, y, acc) in enumerate(problems):
            _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
            _need(x, "X", torch.float32, self.m * k)
            _need(y, "Y", torch.float32, self.m * n)
            if acc is not None:
                _need(acc, "acc", torch.int32, self.m * n)
            arr[i] = Problem(packed.data_ptr(), n, k, x.data_ptr(), y.data_ptr(),
                             None if acc is None else acc.data_ptr())
            self.tensors += [packed, x, y, acc]
        self.array = arr
        self.count = len(problems)
        need = int(lib.bitnet_i2s_quant_gemv_batched_workspace_bytes(arr, self.count, self.m))
        if need == 0:
            raise BitnetError(1, "invalid batch")
        if workspace is None:
            dev = problems[0][0].device
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _need(workspace, "workspace", torch.uint8, need)
        self.device = problems[0][0].device
        for t in self.tensors + [workspace]:
            _same_device(self.device, tensor=t)
        self.workspace = workspace

    def run(self, stream=None) -> None:
        _run(self.device, lib.bitnet_i2s_quant_gemv_batched, self.array, self.count, self.m,
             self.workspace.data_ptr(), self.workspace.numel(), stream=stream)


def bitnet_i2s_quant_gemv_batched(problems, m: int, workspace=None, stream=None) -> None:
    """One call for many independent (packed, N, K, X, Y, acc) problems."""
    BatchedQuantGemv(problems, m, workspace).run(stream)


class QuantGemvChain:
    """Argument block of one bitnet_i2s_quant_gemv_chain call.

    `problems` is a list of (packed, N, K, X, Y, acc_or_None) CUDA tensors
    in dependency order and `stages` their stage numbers (0, then equal or
    one more each time).  A problem whose X is the very tensor (same data
    pointer) that an earlier stage's problem writes as Y reads that output;
    every other X is an external input.  `run()` makes the call (capturable
    in a CUDA graph)."""

    def __init__(self, problems, stages, m: int, workspace: torch.Tensor | None = None):
        self.m = int(m)
        if len(stages) != len(problems):
            raise ValueError("one stage number per problem")
        self.tensors = []
        arr = (Problem * len(problems))()
        for i, (packed, n, k, x, y, acc) in enumerate(problems):
            _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
            _need(x, "X", torch.float32, self.m * k)
            _need(y, "Y", torch.float32, self.m * n)
            if acc is not None:
                _need(acc, "acc", torch.int32, self.m * n)
            arr[i] = Problem(packed.data_ptr(), n, k, x.data_ptr(), y.data_ptr(),
                             None if acc is None else acc.data_ptr())
            self.tensors += [packed, x, y, acc]
        self.array = arr
        self.stages = (ctypes.c_int32 * len(stages))(*[int(v) for v in stages])
        self.count = len(problems)
        need = int(lib.bitnet_i2s_quant_gemv_chain_workspace_bytes(arr, self.stages, self.count,
                                                                   self.m))
        if need == 0:
            raise BitnetError(1, (lib.bitnet_last_error() or b"invalid chain").decode())
        self.device = problems[0][0].device
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        _need(workspace, "workspace", torch.uint8, need)
        for t in self.tensors + [workspace]:
            _same_device(self.device, tensor=t)
        self.workspace = workspace

    def run(self, stream=None) -> None:
        _run(self.device, lib.bitnet_i2s_quant_gemv_chain, self.array, self.stages, self.count,
             self.m, self.workspace.data_ptr(), self.workspace.numel(), stream=stream)


def bitnet_i2s_quant_gemv_chain(problems, stages, m: int, workspace=None, stream=None) -> None:
    """One call for a dependency-ordered chain of (packed, N, K, X, Y, acc)."""
    QuantGemvChain(problems, stages, m, workspace).run(stream)


class QProblem(ctypes.Structure):
    """ctypes mirror of `bitnet_i2s_qproblem`."""
    _fields_ = [("packed", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("Xq", ctypes.c_void_p), ("xs", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("acc_or_null", ctypes.c_void_p)]


class BatchedGemv:
    """Argument block of one bitnet_i2s_gemv_batched call: a list of
    (packed, N, K, Xq, xs, Y, acc_or_None) CUDA tensors, every Xq with M rows.

    `workspace`: True (default) allocates the work counters the call can use,
    None passes no workspace (fixed tile ranges), or a uint8 CUDA tensor."""

    def __init__(self, problems, m: int, workspace=True):
        self.m = int(m)
        self.tensors = []
        arr = (QProblem * len(problems))()
        for i, (packed, n, k, xq, xs, y, acc) in enumerate(problems):
            _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
            _need(xq, "Xq", torch.int8, self.m * k)
            _need(xs, "xs", torch.float32, self.m)
            _need(y, "Y", torch.float32, self.m * n)
            if acc is not None:
                _need(acc, "acc", torch.int32, self.m * n)
            arr[i] = QProblem(packed.data_ptr(), n, k, xq.data_ptr(), xs.data_ptr(), y.data_ptr(),
                              None if acc is None else acc.data_ptr())
            self.tensors += [packed, xq, xs, y, acc]
        self.array = arr
        self.count = len(problems)
        if workspace is True:
            need = int(lib.bitnet_i2s_gemv_batched_workspace_bytes(self.count))
            workspace = torch.empty(need, dtype=torch.uint8, device=problems[0][0].device)
        if workspace is not None:
            _need(workspace, "workspace", torch.uint8)
        self.device = problems[0][0].device
        for t in self.tensors + [workspace]:
            _same_device(self.device, tensor=t)
        self.workspace = workspace

    def run(self, stream=None) -> None:
        ws = self.workspace
        _run(self.device, lib.bitnet_i2s_gemv_batched, self.array, self.count, self.m,
             None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel(),
             stream=stream)


def bitnet_i2s_gemv_batched(problems, m: int, workspace=True, stream=None) -> None:
    """One call for many independent (packed, N, K, Xq, xs, Y, acc) problems."""
    BatchedGemv(problems, m, workspace).run(stream)


def bitnet_i2s_quant_gemv_noalloc(packed, n, k, x, y=None, acc=None, want_acc=False,
                                  stream=None):
    """bitnet_i2s_quant_gemv using the library's static scratch (no workspace)."""
    _need(packed, "packed", torch.uint8, bitnet_i2s_packed_bytes(n, k))
    _need(x, "X", torch.float32)
    m = x.shape[0]
    _need(x, "X", torch.float32, m * k)
    dev = packed.device
    y = torch.empty((m, n), dtype=torch.float32, device=dev) if y is None else y
    _need(y, "Y", torch.float32, m * n)
    if want_acc and acc is None:
        acc = torch.empty((m, n), dtype=torch.int32, device=dev)
    if acc is not None:
        _need(acc, "acc", torch.int32, m * n)
    # The static scratch is chosen by the current device: the call runs with
    # the tensors' device current.
    _same_device(dev, X=x, Y=y, acc=acc)
    _run(dev, lib.bitnet_i2s_quant_gemv_noalloc, _ptr(packed), n, k, _ptr(x), m, _ptr(y),
         _ptr(acc), stream=stream)
    return (y, acc) if acc is not None else y


def bitnet_iq2bn_bytes(n: int, k: int) -> int:
    return int(lib.bitnet_iq2bn_bytes(n, k))


def bitnet_iq1bn_bytes(n: int, k: int) -> int:
    return int(lib.bitnet_iq1bn_bytes(n, k))


def bitnet_iq2bn_pack(w: torch.Tensor, r4: bool = False, out=None, stream=None):
    """fp32 W[N,K] -> uint8 IQ2_BN (or IQ2_BN_R4) tensor."""
    _need(w, "W", torch.float32)
    n, k = w.shape
    nbytes = bitnet_iq2bn_bytes(n, k)
    out = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=w.device) if out is None else out
    _need(out, "out", torch.uint8, nbytes)
    _same_device(w.device, out=out)
    _run(w.device, lib.bitnet_iq2bn_pack, _ptr(w), n, k, int(bool(r4)), _ptr(out), stream=stream)
    return out


def bitnet_iq2bn_dequant_f32(packed, n, k, r4: bool = False, w_out=None, stream=None):
    _need(packed, "packed", torch.uint8, bitnet_iq2bn_bytes(n, k))
    w_out = torch.empty((n, k), dtype=torch.float32, device=packed.device) if w_out is None else w_out
    _need(w_out, "W_out", torch.float32, n * k)
    _same_device(packed.device, W_out=w_out)
    _run(packed.device, lib.bitnet_iq2bn_dequant_f32, _ptr(packed), n, k, int(bool(r4)),
         _ptr(w_out), stream=stream)
    return w_out


def bitnet_iq1bn_pack(w: torch.Tensor, out=None, stream=None):
    """fp32 W[N,K] -> uint8 IQ1_BN tensor."""
    _need(w, "W", torch.float32)
    n, k = w.shape
    nbytes = bitnet_iq1bn_bytes(n, k)
    out = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=w.device) if out is None else out
    _need(out, "out", torch.uint8, nbytes)
    _same_device(w.device, out=out)
    _run(w.device, lib.bitnet_iq1bn_pack, _ptr(w), n, k, _ptr(out), stream=stream)
    return out


def bitnet_iq1bn_dequant_f32(packed, n, k, w_out=None, stream=None):
    _need(packed, "packed", torch.uint8, bitnet_iq1bn_bytes(n, k))
    w_out = torch.empty((n, k), dtype=torch.float32, device=packed.device) if w_out is None else w_out
    _need(w_out, "W_out", torch.float32, n * k)
    _same_device(packed.device, W_out=w_out)
    _run(packed.device, lib.bitnet_iq1bn_dequant_f32, _ptr(packed), n, k, _ptr(w_out),
         stream=stream)
    return w_out


def bitnet_iq2bn_r4_gemv(packed, n, k, xq, xs, y=None, acc=None, want_acc=False, stream=None):
    """Decode matmul (M = Xq.shape[0] in 1..2) on an IQ2_BN_R4 tensor."""
    _need(packed, "packed", torch.uint8, bitnet_iq2bn_bytes(n, k))
    _need(xq, "Xq", torch.int8)
    m = xq.shape[0]
    _need(xq, "Xq", torch.int8, m * k)
    _need(xs, "xs", torch.float32, m)
    dev = packed.device
    y = torch.empty((m, n), dtype=torch.float32, device=dev) if y is None else y
    _need(y, "Y", torch.float32, m * n)
    if want_acc and acc is None:
        acc = torch.empty((m, n), dtype=torch.int32, device=dev)
    if acc is not None:
        _need(acc, "acc", torch.int32, m * n)
    _same_device(dev, Xq=xq, xs=xs, Y=y, acc=acc)
    _run(dev, lib.bitnet_iq2bn_r4_gemv, _ptr(packed), n, k, _ptr(xq), _ptr(xs), m, _ptr(y),
         _ptr(acc), stream=stream)
    return (y, acc) if acc is not None else y


def bitnet_device_status() -> None:
    """Synchronize and raise BitnetError if a device-side wait ran out."""
    _check(lib.bitnet_device_status())


def bitnet_debug_wait_timeout(timeout_ns: int = 1_000_000, stream=None) -> None:
    """Launch one device wait that runs out after timeout_ns (failure-detection check)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _run(dev, lib.bitnet_debug_wait_timeout, int(timeout_ns), stream=stream)


def bitnet_last_error() -> str:
    return lib.bitnet_last_error().decode(errors="replace")
