"""Pins of the oracle's block-64 formats (IQ2_BN, IQ2_BN_R4, IQ1_BN).

"ik_llama.cpp 运行 BitNet b1.58 2B 模型实战" (§5.2, §5.3, §6) fixes: blocks of 64
weights (K a multiple of 64), about 2 bits per weight for IQ2_BN and 1.625
for IQ1_BN, one row quantized at a time, IQ2_BN_R4 = IQ2_BN's blocks in
groups of 4 rows, and an IQ1_BN decode by multiply, add and shift.  It elides
the bits inside a block: the layouts are the oracle's readings (R11-R13), so
byte-level parity with any outside implementation is unpinned.  What the
page fixes, and the mathematics, are pinned here: sizes and bit rates, a
hand-derived worked example of each reading, lossless round trips on
ternary input, R4 as a pure permutation of IQ2_BN, exhaustive trit decoding,
closed forms, and agreement with the pinned I2_S oracle on the same weights.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from i2_mpgemm_b200 import inputs

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "iq2bn_iq1bn_worked_examples.json")))


def ternary_rows(n, k, seed, zero_rows=()):
    """Ternary T with its own scale per row (some rows all zero), and W = T * d."""
    t = inputs.ternary_codes(n, k, seed).numpy()
    g = torch.Generator().manual_seed(seed + 1)
    d = torch.empty(n).uniform_(0.5, 2.0, generator=g).numpy().astype(np.float32)
    for r in zero_rows:
        t[r] = 0
        d[r] = 0.0
    for r in range(n):
        if not np.any(t[r]):
            d[r] = 0.0
    return t, d, (t.astype(np.float32) * d[:, None]).astype(np.float32)


def test_sizes_and_bit_rates():
    for n, k in [(1, 64), (4, 128), (640, 2560), (7, 6912)]:
        assert oracle.iq2bn_bytes(n, k) == n * k // 4 + 4 * n
        assert oracle.iq1bn_bytes(n, k) == n * (k // 64) * 13 + 4 * n
    assert 13 * 8 / 64 == 1.625  # IQ1_BN code bits per weight
    assert 16 * 8 / 64 == 2.0    # IQ2_BN code bits per weight


def test_k_must_be_a_multiple_of_64():
    with pytest.raises(oracle.OracleError):
        oracle.iq2bn_pack(np.zeros((2, 96), np.float32))
    with pytest.raises(oracle.OracleError):
        oracle.iq1bn_pack(np.zeros((2, 96), np.float32))
    with pytest.raises(oracle.OracleError):
        oracle.iq2bn_pack(np.zeros((6, 64), np.float32), r4=True)  # R4 wants N % 4 == 0
    oracle.iq2bn_pack(np.zeros((2, 64), np.float32))  # K = 64 is one block


def test_iq2bn_worked_example():
    ex = GOLD["iq2bn_block"]
    w = np.zeros((1, 64), np.float32)
    for j, v in ex["weights_nonzero"].items():
        w[0, int(j)] = v
    p = oracle.iq2bn_pack(w)
    assert p[:16].tolist() == ex["bytes"]
    assert np.frombuffer(p[16:20].tobytes(), np.float32)[0] == ex["row_scale"]


def test_r4_places_blocks_four_rows_together():
    ex = GOLD["iq2bn_r4_offset"]
    n, k = ex["n"], ex["k"]
    w = np.zeros((n, k), np.float32)
    # a recognisable block: row 5, weights 64..127 (block 1)
    pattern = np.array([1, -1, 0, 1, 1, 0, -1, -1] * 8, np.float32)
    w[ex["row"], 64:128] = pattern
    p2 = oracle.iq2bn_pack(w)
    p4 = oracle.iq2bn_pack(w, r4=True)
    blk = p2[ex["iq2bn_offset"]:ex["iq2bn_offset"] + 16]
    assert not np.all(blk == 0x55)
    assert np.array_equal(p4[ex["r4_offset"]:ex["r4_offset"] + 16], blk)
    # every other block of the R4 tensor is all zeros (code 1)
    rest = np.delete(p4[:n * k // 4], np.arange(ex["r4_offset"], ex["r4_offset"] + 16))
    assert np.all(rest == 0x55)


@pytest.mark.parametrize("n,k", [(4, 64), (8, 256), (12, 640), (640, 2560)])
def test_r4_is_a_permutation_of_iq2bn_blocks(n, k):
    t, d, w = ternary_rows(n, k, 40 + n + k)
    p2 = oracle.iq2bn_pack(w)
    p4 = oracle.iq2bn_pack(w, r4=True)
    nb = k // 64
    b2 = p2[:n * k // 4].reshape(n, nb, 16)
    b4 = p4[:n * k // 4].reshape(n // 4, nb, 4, 16)
    assert np.array_equal(b4.transpose(0, 2, 1, 3).reshape(n, nb, 16), b2)
    assert np.array_equal(p2[n * k // 4:], p4[n * k // 4:])  # same row scales


@pytest.mark.parametrize("n,k", [(1, 64), (4, 128), (13, 640), (64, 2560)])
def test_lossless_round_trips_on_ternary_rows(n, k):
    t, d, w = ternary_rows(n, k, 7 * n + k, zero_rows=(0,) if n > 1 else ())
    for r4 in ([False, True] if n % 4 == 0 else [False]):
        t2, d2 = oracle.iq2bn_unpack(oracle.iq2bn_pack(w, r4=r4), n, k, r4=r4)
        assert np.array_equal(t2, t) and np.array_equal(d2, d)
    t1, d1 = oracle.iq1bn_unpack(oracle.iq1bn_pack(w), n, k)
    assert np.array_equal(t1, t) and np.array_equal(d1, d)
    # the row scale is max |w| of the row
    assert np.array_equal(d, np.abs(w).max(axis=1))


def test_iq1bn_worked_byte():
    ex = GOLD["iq1bn_byte"]
    assert oracle.iq1bn_encode_byte(ex["trits"]) == ex["byte"]
    assert [oracle.iq1bn_trit(ex["byte"], j) for j in range(5)] == ex["trits"]


def test_iq1bn_every_five_trit_byte_decodes_exactly():
    seen = set()
    for v in range(243):
        trits = [(v // 3 ** (4 - j)) % 3 for j in range(5)]
        b = oracle.iq1bn_encode_byte(trits)
        assert 0 <= b <= 255
        assert [oracle.iq1bn_trit(b, j) for j in range(5)] == trits
        seen.add(b)
    assert len(seen) == 243  # distinct bytes


def test_iq1bn_rounding_of_a_nonternary_row_matches_iq2bn():
    g = torch.Generator().manual_seed(3)
    w = torch.randn((5, 192), generator=g).numpy()
    t2, d2 = oracle.iq2bn_unpack(oracle.iq2bn_pack(w), 5, 192)
    t1, d1 = oracle.iq1bn_unpack(oracle.iq1bn_pack(w), 5, 192)
    assert np.array_equal(t1, t2) and np.array_equal(d1, d2)


@pytest.mark.parametrize("sign", [1, -1, 0])
def test_row_scale_matmul_closed_forms(sign):
    n, k, m = 6, 256, 3
    t = np.full((n, k), sign, np.int8)
    d = np.linspace(0.5, 2.0, n).astype(np.float32)
    xq = torch.randint(-127, 128, (m, k), generator=torch.Generator().manual_seed(9),
                       dtype=torch.int8).numpy()
    xs = np.ones(m, np.float32)
    y, acc = oracle.gemm_rows(t, d, xq, xs)
    want = sign * xq.astype(np.int64).sum(axis=1)
    assert np.array_equal(acc, np.repeat(want[:, None], n, axis=1))
    assert np.array_equal(y, (acc.astype(np.float32) * xs[:, None]) * d[None, :])


def test_row_scale_matmul_brute_force_and_agrees_with_i2s_on_one_scale():
    n, k, m = 33, 384, 5
    t = inputs.ternary_codes(n, k, 77).numpy()
    s = np.float32(1.375)
    x = inputs.activations(m, k, 77).numpy()
    xq, xs = oracle.act_quant(x)
    d = np.full(n, s, np.float32)
    y, acc = oracle.gemm_rows(t, d, xq, xs)
    assert np.array_equal(acc, xq.astype(np.int64) @ t.astype(np.int64).T)
    # the same weights as one I2_S tensor with scale s give the same outputs
    y2, acc2 = oracle.gemm(oracle.pack(t.astype(np.float32) * s), n, k, xq, xs)
    assert np.array_equal(acc, acc2) and np.array_equal(y, y2)
