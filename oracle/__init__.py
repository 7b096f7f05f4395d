"""Plain CPU oracle for the I2_S ternary x int8 matmul -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this package.  It wraps ``i2s_oracle.c`` (scalar C,
built with ``-O2 -ffp-contract=off -fno-fast-math``) through ctypes and works
on numpy arrays.  It shares no code with the CUDA library in
``i2_mpgemm_b200``; neither imports the other.

Each function follows one step of the method as the web pages describe it;
the C file lists the pages (by title and section) and every reading taken
where they are silent.  Parity status: every function is pinned by the
``-m "not gpu"`` tests (worked example, closed forms, brute force, error
bounds) except the AbsMean ternarization's choice of eps and tie rule, which
the pages leave open.  The block-64 formats (IQ2_BN, IQ2_BN_R4, IQ1_BN) are
"parity unpinned" in their byte layout: the page elides the bits inside a
block, so the layout is this oracle's reading; what the page and the
arithmetic fix about them (sizes, block of 64, R4 as a 4-row permutation,
lossless round trips, the trit decode, closed forms) is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "i2s_oracle.c")
_LIB = os.path.join(_HERE, "libi2s_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i64, vp, f32, f64 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_float, ctypes.c_double
            lib.i2s_oracle_packed_bytes.restype = ctypes.c_size_t
            lib.i2s_oracle_packed_bytes.argtypes = [i64, i64]
            lib.i2s_oracle_pack.argtypes = [vp, i64, i64, vp]
            lib.i2s_oracle_scale.restype = f32
            lib.i2s_oracle_scale.argtypes = [vp, i64, i64]
            lib.i2s_oracle_unpack.argtypes = [vp, i64, i64, vp, vp]
            lib.i2s_oracle_act_quant.argtypes = [vp, i64, i64, vp, vp]
            lib.i2s_oracle_gemm.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp]
            lib.i2s_oracle_gemm_sampled.argtypes = [vp, i64, i64, vp, vp, i64, vp, vp, i64, vp, vp]
            lib.i2s_oracle_quant_gemm.argtypes = [vp, i64, i64, vp, i64, vp, vp, vp, vp]
            lib.i2s_oracle_ternarize_absmean.argtypes = [vp, i64, f64, vp, vp]
            lib.i2s_oracle_dequant_f32.argtypes = [vp, i64, i64, vp]
            lib.i2s_oracle_iq2bn_bytes.restype = ctypes.c_size_t
            lib.i2s_oracle_iq2bn_bytes.argtypes = [i64, i64]
            lib.i2s_oracle_iq1bn_bytes.restype = ctypes.c_size_t
            lib.i2s_oracle_iq1bn_bytes.argtypes = [i64, i64]
            i32 = ctypes.c_int
            lib.i2s_oracle_iq2bn_pack.argtypes = [vp, i64, i64, i32, vp]
            lib.i2s_oracle_iq2bn_unpack.argtypes = [vp, i64, i64, i32, vp, vp]
            lib.i2s_oracle_iq1bn_pack.argtypes = [vp, i64, i64, vp]
            lib.i2s_oracle_iq1bn_unpack.argtypes = [vp, i64, i64, vp, vp]
            lib.i2s_oracle_iq1bn_encode_byte.argtypes = [vp]
            lib.i2s_oracle_iq1bn_trit.argtypes = [i32, i32]
            lib.i2s_oracle_gemm_rows.argtypes = [vp, vp, i64, i64, vp, vp, i64, vp, vp]
            for name in ("pack", "unpack", "act_quant", "gemm", "gemm_sampled", "quant_gemm",
                         "ternarize_absmean", "dequant_f32", "iq2bn_pack", "iq2bn_unpack",
                         "iq1bn_pack", "iq1bn_unpack", "iq1bn_encode_byte", "iq1bn_trit",
                         "gemm_rows"):
                getattr(lib, "i2s_oracle_" + name).restype = ctypes.c_int
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _check(status: int, what: str) -> None:
    if status != 0:
        raise OracleError(f"oracle {what} failed with status {status}")


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def packed_bytes(n: int, k: int) -> int:
    """Size in bytes of an I2_S tensor of n rows by k columns."""
    return int(_load().i2s_oracle_packed_bytes(n, k))


def pack(w: np.ndarray) -> np.ndarray:
    """fp32 W[N,K] -> uint8 I2_S bytes (codes then the fp32 scale)."""
    w = _c(w, np.float32)
    n, k = w.shape
    out = np.zeros(packed_bytes(n, k), dtype=np.uint8)
    _check(_load().i2s_oracle_pack(_p(w), n, k, _p(out)), "pack")
    return out


def scale(packed: np.ndarray, n: int, k: int) -> float:
    packed = _c(packed, np.uint8)
    return float(_load().i2s_oracle_scale(_p(packed), n, k))


def unpack(packed: np.ndarray, n: int, k: int) -> tuple[np.ndarray, float]:
    """I2_S bytes -> (int8 T[N,K] in {-1,0,+1}, scale)."""
    packed = _c(packed, np.uint8)
    t = np.zeros((n, k), dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    _check(_load().i2s_oracle_unpack(_p(packed), n, k, _p(t), _p(s)), "unpack")
    return t, float(s[0])


def act_quant(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """fp32 X[M,K] -> (int8 Xq[M,K], fp32 xs[M]) by per-token absmax."""
    x = _c(x, np.float32)
    m, k = x.shape
    xq = np.zeros((m, k), dtype=np.int8)
    xs = np.zeros(m, dtype=np.float32)
    _check(_load().i2s_oracle_act_quant(_p(x), m, k, _p(xq), _p(xs)), "act_quant")
    return xq, xs


def gemm(packed: np.ndarray, n: int, k: int, xq: np.ndarray, xs: np.ndarray):
    """(Y fp32 [M,N], acc int32 [M,N]) for packed W[N,K] and Xq[M,K]."""
    packed = _c(packed, np.uint8)
    xq = _c(xq, np.int8)
    xs = _c(xs, np.float32)
    m = xq.shape[0]
    y = np.zeros((m, n), dtype=np.float32)
    acc = np.zeros((m, n), dtype=np.int32)
    _check(_load().i2s_oracle_gemm(_p(packed), n, k, _p(xq), _p(xs), m, _p(y), _p(acc)), "gemm")
    return y, acc


def gemm_sampled(packed, n, k, xq, xs, pos_m, pos_n):
    """The outputs at positions (pos_m[i], pos_n[i]) only."""
    packed = _c(packed, np.uint8)
    xq = _c(xq, np.int8)
    xs = _c(xs, np.float32)
    pm = _c(pos_m, np.int64)
    pn = _c(pos_n, np.int64)
    cnt = pm.shape[0]
    y = np.zeros(cnt, dtype=np.float32)
    acc = np.zeros(cnt, dtype=np.int32)
    _check(_load().i2s_oracle_gemm_sampled(_p(packed), n, k, _p(xq), _p(xs), xq.shape[0],
                                           _p(pm), _p(pn), cnt, _p(y), _p(acc)), "gemm_sampled")
    return y, acc


def quant_gemm(packed, n, k, x):
    """Per-token quantization of x then the matmul: (Y, acc, xq, xs)."""
    packed = _c(packed, np.uint8)
    x = _c(x, np.float32)
    m = x.shape[0]
    y = np.zeros((m, n), dtype=np.float32)
    acc = np.zeros((m, n), dtype=np.int32)
    xq = np.zeros((m, k), dtype=np.int8)
    xs = np.zeros(m, dtype=np.float32)
    _check(_load().i2s_oracle_quant_gemm(_p(packed), n, k, _p(x), m, _p(y), _p(acc), _p(xq),
                                         _p(xs)), "quant_gemm")
    return y, acc, xq, xs


def ternarize_absmean(w: np.ndarray, eps: float = 1e-5) -> tuple[np.ndarray, float]:
    """AbsMean RoundClip ternarization: (W~ * gamma as fp32, gamma as fp64)."""
    w = _c(w, np.float32)
    out = np.zeros_like(w)
    g = np.zeros(1, dtype=np.float64)
    _check(_load().i2s_oracle_ternarize_absmean(_p(w), w.size, float(eps), _p(out), _p(g)),
           "ternarize_absmean")
    return out, float(g[0])


def dequant_f32(packed: np.ndarray, n: int, k: int) -> np.ndarray:
    """Full-tensor I2_S -> fp32 weights (code - 1) * scale."""
    packed = _c(packed, np.uint8)
    out = np.zeros((n, k), dtype=np.float32)
    _check(_load().i2s_oracle_dequant_f32(_p(packed), n, k, _p(out)), "dequant_f32")
    return out


# ---- block-64 formats (IQ2_BN, IQ2_BN_R4, IQ1_BN): readings R11-R14 of the
# C file; their byte layouts are parity unpinned (the page elides them).

def iq2bn_bytes(n: int, k: int) -> int:
    """Size of an IQ2_BN or IQ2_BN_R4 tensor: N*K/4 code bytes + N row scales."""
    return int(_load().i2s_oracle_iq2bn_bytes(n, k))


def iq1bn_bytes(n: int, k: int) -> int:
    """Size of an IQ1_BN tensor: 13 bytes per 64 weights + N row scales."""
    return int(_load().i2s_oracle_iq1bn_bytes(n, k))


def iq2bn_pack(w: np.ndarray, r4: bool = False) -> np.ndarray:
    """fp32 W[N,K] -> IQ2_BN (or IQ2_BN_R4) bytes."""
    w = _c(w, np.float32)
    n, k = w.shape
    out = np.zeros(iq2bn_bytes(n, k), dtype=np.uint8)
    _check(_load().i2s_oracle_iq2bn_pack(_p(w), n, k, int(r4), _p(out)), "iq2bn_pack")
    return out


def iq2bn_unpack(p: np.ndarray, n: int, k: int, r4: bool = False):
    """IQ2_BN (or IQ2_BN_R4) bytes -> (int8 T[N,K], fp32 row scales d[N])."""
    p = _c(p, np.uint8)
    t = np.zeros((n, k), dtype=np.int8)
    d = np.zeros(n, dtype=np.float32)
    _check(_load().i2s_oracle_iq2bn_unpack(_p(p), n, k, int(r4), _p(t), _p(d)), "iq2bn_unpack")
    return t, d


def iq1bn_pack(w: np.ndarray) -> np.ndarray:
    """fp32 W[N,K] -> IQ1_BN bytes."""
    w = _c(w, np.float32)
    n, k = w.shape
    out = np.zeros(iq1bn_bytes(n, k), dtype=np.uint8)
    _check(_load().i2s_oracle_iq1bn_pack(_p(w), n, k, _p(out)), "iq1bn_pack")
    return out


def iq1bn_unpack(p: np.ndarray, n: int, k: int):
    """IQ1_BN bytes -> (int8 T[N,K], fp32 row scales d[N])."""
    p = _c(p, np.uint8)
    t = np.zeros((n, k), dtype=np.int8)
    d = np.zeros(n, dtype=np.float32)
    _check(_load().i2s_oracle_iq1bn_unpack(_p(p), n, k, _p(t), _p(d)), "iq1bn_unpack")
    return t, d


def iq1bn_encode_byte(trits) -> int:
    """The IQ1_BN byte of five trits (each 0, 1 or 2; the first most significant)."""
    a = _c(np.asarray(trits), np.int32)
    return int(_load().i2s_oracle_iq1bn_encode_byte(_p(a)))


def iq1bn_trit(byte: int, j: int) -> int:
    """Trit j (0..4) of an IQ1_BN byte, by multiply and shift."""
    return int(_load().i2s_oracle_iq1bn_trit(int(byte), int(j)))


def gemm_rows(t: np.ndarray, d: np.ndarray, xq: np.ndarray, xs: np.ndarray):
    """(Y, acc) of ternary T[N,K] with row scales d[N] and Xq[M,K]."""
    t = _c(t, np.int8)
    d = _c(d, np.float32)
    xq = _c(xq, np.int8)
    xs = _c(xs, np.float32)
    n, k = t.shape
    m = xq.shape[0]
    y = np.zeros((m, n), dtype=np.float32)
    acc = np.zeros((m, n), dtype=np.int32)
    _check(_load().i2s_oracle_gemm_rows(_p(t), _p(d), n, k, _p(xq), _p(xs), m, _p(y), _p(acc)),
           "gemm_rows")
    return y, acc


def quant_gemm_chain(problems):
    """A dependency chain of fused problems, run one after the other.

    `problems` is a list in order; each entry is (packed, n, k, src) where
    `src` is either an fp32 [m, k] array (an external input) or the index of
    an earlier entry whose output Y [m, n_src] (n_src == k) is the input.
    This is the seven projections of a BitNet b1.58 layer in a decode step
    ("BitNet Inference Preprocessing: Converting Hugging Face Checkpoints to
    I2S GGUF", The Two-Stage BitNet Inference Preprocessing Pipeline, names
    them) where each quantizes its input per token before the ternary matmul
    ("LLM Quantization Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026",
    section 5): nothing but quant_gemm applied in order, each on the fp32
    output the one it reads has produced.  Returns [(Y, acc, xq, xs)]."""
    out = []
    for i, (packed, n, k, src) in enumerate(problems):
        if isinstance(src, (int, np.integer)):
            if not 0 <= src < i:
                raise ValueError(f"problem {i} reads problem {src}, which does not come before it")
            x = out[src][0]
            if x.shape[1] != k:
                raise ValueError(f"problem {i}: K={k} but its input has {x.shape[1]} columns")
        else:
            x = src
        out.append(quant_gemm(packed, n, k, x))
    return out
