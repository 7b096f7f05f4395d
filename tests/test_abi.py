"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before touching CUDA.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"BITNET_API\s+[\w\s\*]+?\b(bitnet_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def i2s():
    from i2_mpgemm_b200 import build
    build.build()
    from i2_mpgemm_b200 import i2s as mod
    return mod


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("bitnet_i2s_packed_bytes", "bitnet_i2s_pack", "bitnet_act_quant_i8",
                     "bitnet_i2s_gemv", "bitnet_i2s_gemm", "bitnet_i2s_quant_gemv",
                     "bitnet_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(i2s):
    lib = ctypes.CDLL(i2s.LIB_PATH)
    names = declared_functions()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # the binding wraps exactly the declared functions
    assert set(i2s.SIGNATURES) == names


def test_size_helpers(i2s):
    assert i2s.bitnet_i2s_packed_bytes(640, 2560) == 640 * 2560 // 4 + 4
    assert i2s.bitnet_i2s_packed_bytes(1, 100) == 0
    assert i2s.bitnet_i2s_packed_bytes(0, 128) == 0
    ws = i2s.bitnet_i2s_quant_gemv_workspace_bytes(3, 256)
    assert ws >= 3 * 256 + 3 * 4 and ws % 256 == 0
    assert i2s.bitnet_i2s_quant_gemv_workspace_bytes(0, 256) == 0


def _call(i2s, name, *args):
    return getattr(i2s.lib, name)(*args)


A = 1 << 20  # a 256-byte aligned fake address: never dereferenced, checks fail first


def test_matmul_argument_errors_on_host(i2s):
    for fn in ("bitnet_i2s_gemv", "bitnet_i2s_gemm"):
        # null pointers
        assert _call(i2s, fn, None, 8, 128, A, A, 1, A, None, None) == 1
        assert _call(i2s, fn, A, 8, 128, None, A, 1, A, None, None) == 1
        assert _call(i2s, fn, A, 8, 128, A, None, 1, A, None, None) == 1
        assert _call(i2s, fn, A, 8, 128, A, A, 1, None, None, None) == 1
        # shapes
        assert _call(i2s, fn, A, 0, 128, A, A, 1, A, None, None) == 2
        assert _call(i2s, fn, A, 8, 128, A, A, 0, A, None, None) == 2
        assert _call(i2s, fn, A, 8, 100, A, A, 1, A, None, None) == 2
        assert _call(i2s, fn, A, 8, 0, A, A, 1, A, None, None) == 2
        assert _call(i2s, fn, A, 8, 262144, A, A, 1, A, None, None) == 2
        # alignment
        assert _call(i2s, fn, A + 8, 8, 128, A, A, 1, A, None, None) == 3
        assert _call(i2s, fn, A, 8, 128, A + 4, A, 1, A, None, None) == 3
        assert _call(i2s, fn, A, 8, 128, A, A, 1, A + 2, None, None) == 3
        assert "aligned" in i2s.bitnet_last_error()
    # decode entry is limited to 64 tokens
    assert _call(i2s, "bitnet_i2s_gemv", A, 8, 128, A, A, 65, A, None, None) == 2


def test_pack_and_quant_argument_errors_on_host(i2s):
    assert _call(i2s, "bitnet_i2s_pack", None, 4, 128, A, None) == 1
    assert _call(i2s, "bitnet_i2s_pack", A, 4, 96, A, None) == 2
    assert _call(i2s, "bitnet_i2s_pack", A + 4, 4, 128, A, None) == 3
    assert _call(i2s, "bitnet_act_quant_i8", A, 2, 24, A, A, None) == 2
    assert _call(i2s, "bitnet_act_quant_i8", A, 0, 32, A, A, None) == 2
    assert _call(i2s, "bitnet_act_quant_i8", A + 4, 2, 32, A, A, None) == 3
    assert _call(i2s, "bitnet_act_quant_i8", A, 2, 32, None, A, None) == 1
    fn = "bitnet_i2s_quant_gemv"
    need = i2s.bitnet_i2s_quant_gemv_workspace_bytes(2, 128)
    assert _call(i2s, fn, A, 8, 128, A, 2, A, None, None, need, None) == 1
    assert _call(i2s, fn, A, 8, 128, A, 2, A, None, A + 16, need, None) == 3
    assert _call(i2s, fn, A, 8, 128, A, 2, A, None, A, need - 1, None) == 1
    assert "workspace" in i2s.bitnet_last_error()


def test_product_package_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "i2_mpgemm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
                assert "i2s_oracle" not in text, f


def test_debug_wait_timeout_rejects_out_of_range_on_host(i2s):
    assert i2s.lib.bitnet_debug_wait_timeout(10, None) == 1
    assert i2s.lib.bitnet_debug_wait_timeout(10 ** 10, None) == 1


def test_gemv_batched_workspace_checks_on_host(i2s):
    assert i2s.bitnet_i2s_gemv_batched_workspace_bytes(0) == 0
    one = i2s.bitnet_i2s_gemv_batched_workspace_bytes(1)
    assert one >= 4 and one % 256 == 0
    assert i2s.bitnet_i2s_gemv_batched_workspace_bytes(161) >= 8

    class QP(ctypes.Structure):
        _fields_ = [("packed", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                    ("Xq", ctypes.c_void_p), ("xs", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                    ("acc_or_null", ctypes.c_void_p)]
    arr = (QP * 1)(QP(A, 8, 128, A, A, A, None))
    fn = i2s.lib.bitnet_i2s_gemv_batched
    assert fn(arr, 1, 1, A + 16, one, None) == 3
    assert fn(arr, 1, 1, A, one - 1, None) == 1
    assert "workspace" in i2s.bitnet_last_error()


def _align(v):
    return (v + 255) // 256 * 256


def test_batched_workspace_layout(i2s):
    """Activation slots (M x K int8 and M scales, each 256-byte aligned), then
    the decode tail: one work counter per decode launch and, for up to two
    tokens, per launch 512 x 4 split arrival counters and 512 x 128 x M
    split partial sums."""
    ks = [2560, 2560, 2560, 2560, 2560, 2560, 6912] * 30
    arr = (i2s.Problem * len(ks))()
    for i, k in enumerate(ks):
        arr[i] = i2s.Problem(A, 640, k, A, A, None)
    launches = -(-len(ks) // 160) + 1  # one more: long-K and short-K problems launch apart
    for m in (1, 2, 3, 16):
        slots = sum(_align(m * k) + _align(4 * m) for k in ks)
        tail = _align(4 * (launches + (launches * 512 * 4 if m <= 2 else 0)))
        if m <= 2:
            tail += _align(4 * launches * 512 * 128 * m)
        need = i2s.lib.bitnet_i2s_quant_gemv_batched_workspace_bytes(arr, len(ks), m)
        assert need == slots + tail, m
    assert i2s.lib.bitnet_i2s_quant_gemv_batched_workspace_bytes(arr, 0, 1) == 0
    # the single fused call uses the batched layout for one problem
    one = (i2s.Problem * 1)()
    one[0] = i2s.Problem(A, 640, 2560, A, A, None)
    for m in (1, 2, 5, 127):
        assert (i2s.bitnet_i2s_quant_gemv_workspace_bytes(m, 2560) ==
                i2s.lib.bitnet_i2s_quant_gemv_batched_workspace_bytes(one, 1, m))
    # the pre-quantized batched call sizes its split area for two tokens
    assert i2s.bitnet_i2s_gemv_batched_workspace_bytes(210) == (
        _align(4 * (launches + launches * 512 * 4)) + _align(4 * launches * 512 * 128 * 2))


def _chain(i2s, specs, m):
    """(descriptor array, stage array) of (N, K, X, Y, stage) fake-address specs."""
    arr = (i2s.Problem * len(specs))()
    stages = (ctypes.c_int32 * len(specs))()
    for i, (n, k, x, y, st) in enumerate(specs):
        arr[i] = i2s.Problem(A, n, k, x, y, None)
        stages[i] = st
    return arr, stages


def _chain_bytes(i2s, specs, m):
    arr, stages = _chain(i2s, specs, m)
    return i2s.lib.bitnet_i2s_quant_gemv_chain_workspace_bytes(arr, stages, len(specs), m)


def test_chain_workspace_layout(i2s):
    """Per-problem done counters (256 bytes apart), per-row-tile counters, then M x N
    accumulators per problem (64-int aligned): all zeroed; then two scales
    per problem."""
    Y = 1 << 30  # outputs far apart
    specs = [(2560, 2560, A, Y, 0), (640, 2560, A, Y + (1 << 24), 0),
             (2560, 2560, Y, Y + (2 << 24), 1), (6912, 2560, Y + (2 << 24), Y + (3 << 24), 2),
             (2560, 6912, Y + (3 << 24), Y + (4 << 24), 3)]
    for m in (1, 2):
        ints = 64 * len(specs) + sum(-(-n // 128) for n, *_ in specs)
        ints = -(-ints // 64) * 64 + sum(-(-m * n // 64) * 64 for n, *_ in specs)
        want = _align(4 * ints) + _align(8 * len(specs))
        assert _chain_bytes(i2s, specs, m) == want, m
    # 130 problems (two launches)
    many = [(128, 128, A, Y + i * 4096, 0) for i in range(130)]
    ints = 64 * 130 + 130
    ints = -(-ints // 64) * 64 + 130 * 128
    assert _chain_bytes(i2s, many, 1) == _align(4 * ints) + _align(8 * 130)


def test_chain_argument_errors_on_host(i2s):
    Y = 1 << 30
    ok = [(256, 128, A, Y, 0), (128, 256, Y, Y + 4096, 1)]
    assert _chain_bytes(i2s, ok, 1) > 0
    bad = {
        "three tokens": (ok, 3),
        "stage not from 0": ([(256, 128, A, Y, 1)], 1),
        "stage jumps": ([(256, 128, A, Y, 0), (128, 256, Y, Y + 4096, 2)], 1),
        "stage falls": ([(256, 128, A, Y, 0), (128, 256, A, Y + 4096, 1),
                         (128, 128, A, Y + 8192, 0)], 1),
        "reads the same stage": ([(256, 128, A, Y, 0), (128, 256, Y, Y + 4096, 0)], 1),
        "reads a later stage": ([(128, 256, Y, Y + 4096, 0), (256, 128, A, Y, 1)], 1),
        "K differs from the source's N": ([(384, 128, A, Y, 0), (128, 256, Y, Y + 4096, 1)], 1),
        "input inside an output": ([(256, 128, A, Y, 0), (128, 128, Y + 512, Y + 4096, 1)], 1),
        "input straddles an output": ([(256, 128, A, Y + 512, 0), (128, 256, Y, Y + 8192, 1)], 1),
        "outputs overlap": ([(256, 128, A, Y, 0), (256, 128, A, Y + 512, 0)], 1),
        "unaligned input": ([(256, 128, A + 4, Y, 0)], 1),
    }
    for what, (specs, m) in bad.items():
        assert _chain_bytes(i2s, specs, m) == 0, what
        arr, stages = _chain(i2s, specs, m)
        st = i2s.lib.bitnet_i2s_quant_gemv_chain(arr, stages, len(specs), m, A, 1 << 30, None)
        assert st in (1, 2, 3), (what, st)
    arr, stages = _chain(i2s, ok, 1)
    need = _chain_bytes(i2s, ok, 1)
    assert i2s.lib.bitnet_i2s_quant_gemv_chain(arr, stages, 2, 1, A, need - 1, None) == 1
    assert i2s.lib.bitnet_i2s_quant_gemv_chain(arr, stages, 2, 1, A + 16, need, None) == 3
    assert i2s.lib.bitnet_i2s_quant_gemv_chain(arr, stages, 2, 1, None, need, None) == 1
    assert i2s.lib.bitnet_i2s_quant_gemv_chain(arr, None, 2, 1, A, need, None) == 1
