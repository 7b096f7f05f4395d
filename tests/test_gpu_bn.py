"""GPU parity of the block-64 formats (IQ2_BN, IQ2_BN_R4, IQ1_BN) against the
oracle: packed bytes and dequantized weights bit-exact, the IQ2_BN_R4 decode
matmul's int32 accumulators bit-exact and fp32 outputs within 1e-5 relative
error.  The layouts are the oracle's readings of a page that elides them, so
this is parity with the oracle, not with an outside format."""
import numpy as np
import pytest
import torch

import oracle
from i2_mpgemm_b200 import inputs
from tests.parity import assert_acc_equal, assert_y_close, guarded_empty, guards_intact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def i2s():
    from i2_mpgemm_b200 import i2s as mod
    return mod


def row_weights(n, k, seed, zero_rows=True):
    t = inputs.ternary_codes(n, k, seed).numpy()
    g = torch.Generator().manual_seed(seed + 1)
    d = torch.empty(n).uniform_(0.5, 2.0, generator=g).numpy().astype(np.float32)
    if zero_rows and n > 2:
        t[1] = 0
    return torch.from_numpy((t.astype(np.float32) * d[:, None]).astype(np.float32))


SHAPES = [(4, 64), (8, 128), (12, 640), (640, 2560), (2560, 6912), (28, 8192)]


@pytest.mark.parametrize("n,k", SHAPES)
@pytest.mark.parametrize("r4", [False, True])
def test_iq2bn_pack_and_dequant_are_exact(i2s, n, k, r4):
    w = row_weights(n, k, 100 + n + k)
    out, buf = guarded_empty((i2s.bitnet_iq2bn_bytes(n, k),), torch.uint8)
    i2s.bitnet_iq2bn_pack(w.cuda(), r4=r4, out=out)
    ref = oracle.iq2bn_pack(w.numpy(), r4=r4)
    assert np.array_equal(out.cpu().numpy(), ref)
    assert guards_intact(buf)
    back = i2s.bitnet_iq2bn_dequant_f32(out, n, k, r4=r4).cpu().numpy()
    assert np.array_equal(back, w.numpy())  # lossless on ternary rows


def test_iq2bn_pack_of_arbitrary_weights(i2s):
    n, k = 9, 384
    w = torch.randn((n, k), generator=torch.Generator().manual_seed(5))
    w[:, 3] = 0.5 * w.abs().max(dim=1).values  # exact ties at half the row's scale
    got = i2s.bitnet_iq2bn_pack(w.cuda()).cpu().numpy()
    assert np.array_equal(got, oracle.iq2bn_pack(w.numpy()))


@pytest.mark.parametrize("n,k", [(4, 64), (12, 640), (640, 2560), (100, 6912)])
def test_iq1bn_pack_and_dequant_are_exact(i2s, n, k):
    w = row_weights(n, k, 300 + n + k)
    out, buf = guarded_empty((i2s.bitnet_iq1bn_bytes(n, k),), torch.uint8)
    i2s.bitnet_iq1bn_pack(w.cuda(), out=out)
    assert np.array_equal(out.cpu().numpy(), oracle.iq1bn_pack(w.numpy()))
    assert guards_intact(buf)
    back = i2s.bitnet_iq1bn_dequant_f32(out, n, k).cpu().numpy()
    assert np.array_equal(back, w.numpy())


@pytest.mark.parametrize("m", [1, 2])
@pytest.mark.parametrize("n,k", [(4, 64), (12, 640), (640, 2560), (2560, 6912), (1028, 8192)])
def test_iq2bn_r4_gemv_matches_oracle(i2s, m, n, k):
    w = row_weights(n, k, 500 + n + k + m)
    x = inputs.activations(m, k, 500 + n, outliers=True)
    xq, xs = oracle.act_quant(x.numpy())
    p4 = oracle.iq2bn_pack(w.numpy(), r4=True)
    t, d = oracle.iq2bn_unpack(p4, n, k, r4=True)
    y_ref, acc_ref = oracle.gemm_rows(t, d, xq, xs)
    y, yb = guarded_empty((m, n), torch.float32)
    acc, ab = guarded_empty((m, n), torch.int32)
    i2s.bitnet_iq2bn_r4_gemv(torch.from_numpy(p4).cuda(), n, k, torch.from_numpy(xq).cuda(),
                             torch.from_numpy(xs).cuda(), y=y, acc=acc)
    assert_acc_equal(acc.cpu().numpy(), acc_ref)
    assert_y_close(y.cpu().numpy(), y_ref)
    assert guards_intact(yb) and guards_intact(ab)


def test_i2s_to_iq2bn_r4_through_f32_keeps_the_matmul(i2s):
    """The page's conversion chain I2_S -> f32 -> IQ2_BN_R4 on the GPU: the
    matmul on the converted tensor gives the I2_S matmul's results (every
    row of these weights has a nonzero, so each row scale is the tensor's)."""
    n, k, m = 640, 2560, 1
    w, t, s = inputs.ternary_weights(n, k, 42)
    assert np.all(np.any(t.numpy() != 0, axis=1))
    packed = i2s.bitnet_i2s_pack(w.cuda())
    w32 = i2s.bitnet_i2s_dequant_f32(packed, n, k)
    r4 = i2s.bitnet_iq2bn_pack(w32, r4=True)
    x = inputs.activations(m, k, 42).cuda()
    xq, xs = i2s.bitnet_act_quant_i8(x)
    y1, a1 = i2s.bitnet_i2s_gemv(packed, n, k, xq, xs, want_acc=True)
    y2, a2 = i2s.bitnet_iq2bn_r4_gemv(r4, n, k, xq, xs, want_acc=True)
    assert torch.equal(a1, a2) and torch.equal(y1, y2)
