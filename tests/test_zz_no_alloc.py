"""bitnet_i2s_quant_gemv_noalloc: the fused call for callers that cannot allocate.

Some callers cannot give the library device scratch -- a plug-in handed only
raw input and output pointers by a framework that owns every allocation, or
a latency-critical loop that must never enter the CUDA allocator.  This entry
point keeps its scratch in a fixed 1 MiB array of the library's device image
instead of taking a workspace.  These tests call it through the C ABI several
times in a row (larger shape first, so anything a call left in the shared
array would show up in the next one) and compare each result with the CPU
oracle and with the workspace entry point, bitnet_i2s_quant_gemv: int32
accumulators equal, fp32 outputs within 1e-5 relative error.  The largest
shape that fits the array is accepted and computed correctly; one token more
is refused.  The file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from tests.parity import assert_acc_equal, assert_y_close

A = 1 << 20  # an aligned fake address: the size check fails before any use
SCRATCH_BYTES = 1 << 20  # the static array's size, as the header states


@pytest.fixture(scope="module")
def i2s():
    from i2_mpgemm_b200 import build
    build.build()
    from i2_mpgemm_b200 import i2s as mod
    return mod


def largest_m(i2s, k):
    """The most tokens of length k whose scratch fits the static array."""
    m = 1
    while i2s.bitnet_i2s_quant_gemv_workspace_bytes(m + 1, k) <= SCRATCH_BYTES:
        m += 1
    return m


def test_noalloc_rejects_shapes_beyond_its_static_scratch(i2s):
    # 1024 tokens x 8192 needs 8 MiB of scratch, more than the fixed 1 MiB.
    st = i2s.lib.bitnet_i2s_quant_gemv_noalloc(A, 8, 8192, A, 1024, A, None, None)
    assert st == 2
    assert "static scratch" in i2s.bitnet_last_error()
    # one token more than the largest shape that fits is refused as well
    m = largest_m(i2s, 8192)
    st = i2s.lib.bitnet_i2s_quant_gemv_noalloc(A, 8, 8192, A, m + 1, A, None, None)
    assert st == 2
    assert "static scratch" in i2s.bitnet_last_error()


def _call(i2s, packed, n, k, x, m):
    y = torch.full((m, n), float("nan"), device="cuda")
    acc = torch.full((m, n), -1, dtype=torch.int32, device="cuda")
    st = i2s.lib.bitnet_i2s_quant_gemv_noalloc(packed.data_ptr(), n, k, x.data_ptr(), m,
                                               y.data_ptr(), acc.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream)
    assert st == 0, i2s.bitnet_last_error()
    torch.cuda.synchronize()
    return y, acc


@pytest.mark.gpu
def test_noalloc_matches_the_oracle_and_the_workspace_entry_on_consecutive_calls(i2s):
    import oracle
    from i2_mpgemm_b200 import inputs
    m_max = largest_m(i2s, 8192)
    # (tokens, rows, K): the largest shape that fits the array (tensor-core
    # path), then the tensor-core path, the integer-ALU path, the tensor-core
    # path again, and the ALU path with two tokens.
    cases = [(m_max, 130, 8192, 10), (16, 300, 8192, 11), (1, 640, 2560, 12), (3, 130, 640, 13),
             (2, 257, 1024, 14)]
    for m, n, k, seed in cases:
        w, _, _ = inputs.ternary_weights(n, k, seed)
        x_h = inputs.activations(m, k, seed, outliers=True)
        x = x_h.cuda()
        packed = i2s.bitnet_i2s_pack(w.cuda())
        what = f"M={m} {n}x{k}"
        y_ws, acc_ws = i2s.bitnet_i2s_quant_gemv(packed, n, k, x, want_acc=True)
        y, acc = _call(i2s, packed, n, k, x, m)
        y_ref, acc_ref, _, _ = oracle.quant_gemm(oracle.pack(w.numpy()), n, k, x_h.numpy())
        assert_acc_equal(acc.cpu().numpy(), acc_ref, what)
        assert_y_close(y.cpu().numpy(), y_ref, what)
        assert_acc_equal(acc.cpu().numpy(), acc_ws.cpu().numpy(), what)
        assert_y_close(y.cpu().numpy(), y_ws.cpu().numpy(), what)
        assert np.isfinite(y.cpu().numpy()).all()
    i2s.bitnet_device_status()
