"""Pins of the oracle's dependency chain (quant_gemm applied in order, each
problem on the fp32 output of the one it reads) against facts that hold
outside the oracle: re-quantizing an identity layer's output gives back the
same int8 codes, an all-(+1) layer has a closed form at every stage, and each
problem reads the output it names (not the previous one, not its int32
accumulators, not its int8 codes).  A slip in the composition (a wrong
source index, the accumulators or codes passed on instead of Y) fails one of
them.
"""
import numpy as np
import pytest

import oracle


def _x(m, k, seed):
    return np.random.default_rng(seed).standard_normal((m, k)).astype(np.float32)


@pytest.mark.parametrize("m", [1, 2])
def test_identity_chain_keeps_the_codes(m):
    """W = I (scale 1): Y = xq * xs, whose absmax is 127 * xs, so each next
    stage quantizes it back to the very same codes, with the same scale up
    to the rounding of 127 * xs / 127."""
    k = 256
    eye = oracle.pack(np.eye(k, dtype=np.float32))
    x = _x(m, k, 3)
    out = oracle.quant_gemm_chain([(eye, k, k, x), (eye, k, k, 0), (eye, k, k, 1)])
    xq0, xs0 = oracle.act_quant(x)
    for y, acc, xq, xs in out:
        assert np.array_equal(xq, xq0)
        assert np.allclose(xs, xs0, rtol=2.0 ** -22, atol=0.0)
        assert np.array_equal(acc, xq0.astype(np.int32))
        assert np.array_equal(y, (xq0.astype(np.float32) * xs[:, None]).astype(np.float32))


def test_all_plus_one_chain_closed_form():
    """Every weight +1 with scale s: each output row is constant,
    c = ((sum xq) * xs) * s, so the next stage's codes are all sign(c) * 127,
    its scale |c| / 127 and its sums 127 * K * sign(c)."""
    n0, k0, n1 = 384, 256, 128
    s0, s1 = np.float32(0.75), np.float32(1.5)
    w0 = oracle.pack(np.full((n0, k0), s0, dtype=np.float32))
    w1 = oracle.pack(np.full((n1, n0), s1, dtype=np.float32))
    x = _x(2, k0, 11)
    out = oracle.quant_gemm_chain([(w0, n0, k0, x), (w1, n1, n0, 0)])
    xq, xs = oracle.act_quant(x)
    tot = xq.astype(np.int64).sum(axis=1)
    c = ((tot.astype(np.float32) * xs).astype(np.float32) * s0).astype(np.float32)
    assert np.array_equal(out[0][0], np.repeat(c[:, None], n0, axis=1))
    sign = np.sign(c).astype(np.int64)
    assert np.array_equal(out[1][2], np.repeat((sign * 127)[:, None], n0, axis=1).astype(np.int8))
    xs1 = (np.abs(c) / np.float32(127)).astype(np.float32)
    assert np.array_equal(out[1][3], xs1)
    assert np.array_equal(out[1][1], np.repeat((sign * 127 * n0)[:, None], n1, axis=1))
    y1 = (((sign * 127 * n0).astype(np.float32) * xs1).astype(np.float32) * s1).astype(np.float32)
    assert np.array_equal(out[1][0], np.repeat(y1[:, None], n1, axis=1))


def test_each_problem_reads_the_output_it_names():
    """q and k read x; o (identity weights) reads k, not the problem just
    before it: o's sums are the codes of k's fp32 output."""
    k = 256
    rng = np.random.default_rng(5)
    wq = oracle.pack(rng.integers(-1, 2, (k, k)).astype(np.float32))
    wk = oracle.pack(rng.integers(-1, 2, (k, k)).astype(np.float32) * np.float32(0.5))
    eye = oracle.pack(np.eye(k, dtype=np.float32))
    x = _x(1, k, 7)
    out = oracle.quant_gemm_chain([(wq, k, k, x), (wk, k, k, x), (eye, k, k, 1), (eye, k, k, 0)])
    for o, src in ((2, 1), (3, 0)):
        xq_src, _ = oracle.act_quant(out[src][0])
        assert np.array_equal(out[o][1], xq_src.astype(np.int32))
    assert not np.array_equal(out[2][1], out[3][1])


def test_chain_rejects_forward_references_and_shape_mismatch():
    k = 128
    eye = oracle.pack(np.eye(k, dtype=np.float32))
    with pytest.raises(ValueError):
        oracle.quant_gemm_chain([(eye, k, k, 0)])
    wide = oracle.pack(np.zeros((256, k), dtype=np.float32))
    with pytest.raises(ValueError):
        oracle.quant_gemm_chain([(wide, 256, k, _x(1, k, 1)), (eye, k, k, 0)])
