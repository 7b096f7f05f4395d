"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it cannot agree with by
construction: bytes worked out by hand from the pages' format description
(tests/golden), closed forms of the ternary contraction, brute force with an
independent integer matmul on the generator's ternary matrix (never on the
oracle's own unpack), and error bounds of rounding.  A plausible slip in the
oracle (a wrong shift, group or byte index, a swapped code map, a transposed
operand, a dropped subtraction or epsilon, round-half-away instead of
half-even, a wrong divisor or association in the scales) fails at least one
of them.  The clamps in the float-to-ternary rule and in the activation
quantizer cannot change any result (|w/max|w|| <= 1 and |x*127/amax| rounds
to at most 127), so no test can tell them apart from their absence.
"""
import json
import os

import numpy as np
import pytest

import oracle
from i2_mpgemm_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _weights_from_example(ex):
    w = np.zeros((ex["n"], ex["k"]), dtype=np.float32)
    for r, c, v in ex["nonzero"]:
        w[r, c] = v
    return w * np.float32(ex["scale"])


# --- pack: hand-derived bytes ------------------------------------------------

@pytest.mark.parametrize("idx", [0, 1])
def test_pack_matches_hand_derived_bytes(idx):
    ex = _load("i2s_pack_worked_examples.json")["examples"][idx]
    got = oracle.pack(_weights_from_example(ex))
    assert got.tobytes().hex() == ex["expected_hex"]


@pytest.mark.parametrize("idx", [0, 1])
def test_unpack_of_hand_derived_bytes(idx):
    ex = _load("i2s_pack_worked_examples.json")["examples"][idx]
    packed = np.frombuffer(bytes.fromhex(ex["expected_hex"]), dtype=np.uint8)
    t, s = oracle.unpack(packed, ex["n"], ex["k"])
    want = np.zeros((ex["n"], ex["k"]), dtype=np.int8)
    for r, c, v in ex["nonzero"]:
        want[r, c] = v
    assert np.array_equal(t, want)
    assert s == np.float32(ex["scale"])


def test_packed_size_is_two_bits_per_weight_plus_scale():
    for n, k in [(1, 128), (640, 2560), (6912, 2560), (2560, 6912)]:
        assert oracle.packed_bytes(n, k) == n * k // 4 + 4


def test_unpack_rejects_code_three():
    packed = np.full(32 + 4, 0x55, dtype=np.uint8)
    packed[7] = 0x57  # group 3 of byte 7 holds code 3, which no weight maps to
    with pytest.raises(oracle.OracleError):
        oracle.unpack(packed, 1, 128)


def test_pack_rejects_k_not_multiple_of_block():
    with pytest.raises(oracle.OracleError):
        oracle.pack(np.zeros((2, 64), dtype=np.float32))


# --- pack: losslessness and the scale ----------------------------------------

@pytest.mark.parametrize("n,k,seed", [(1, 128, 0), (3, 256, 1), (7, 384, 2), (33, 128, 3),
                                      (5, 640, 4), (64, 1024, 5)])
def test_round_trip_is_lossless_on_ternary_times_scale(n, k, seed):
    w, t, s = inputs.ternary_weights(n, k, seed)
    packed = oracle.pack(w.numpy())
    t2, s2 = oracle.unpack(packed, n, k)
    assert np.array_equal(t2, t.numpy())
    if np.any(t.numpy() != 0):
        assert s2 == np.float32(s)


def test_scale_is_max_abs_of_arbitrary_weights():
    rng = np.random.default_rng(11)
    w = rng.standard_normal((9, 384)).astype(np.float32)
    packed = oracle.pack(w)
    assert oracle.scale(packed, 9, 384) == np.max(np.abs(w))


def test_all_zero_tensor_stores_zero_scale_and_zero_codes():
    packed = oracle.pack(np.zeros((3, 128), dtype=np.float32))
    assert np.all(packed[:-4] == 0x55)
    t, s = oracle.unpack(packed, 3, 128)
    assert s == 0.0 and not t.any()


def test_float_to_ternary_rule_on_clear_margins():
    # s = 2 (the max); 0.49*s -> 0, 0.51*s -> +1, -0.51*s -> -1, 1.0*s -> +1.
    w = np.zeros((1, 128), dtype=np.float32)
    vals = {0: 2.0, 1: 0.98, 2: 1.02, 3: -1.02, 4: -0.98, 5: -2.0, 6: 0.0, 7: 1.5}
    for c, v in vals.items():
        w[0, c] = v
    t, s = oracle.unpack(oracle.pack(w), 1, 128)
    assert s == 2.0
    assert list(t[0, :8]) == [1, 0, 1, -1, 0, -1, 0, 1]


# --- contraction: closed forms and brute force --------------------------------

def _xq_random(m, k, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(-127, 128, size=(m, k), dtype=np.int64).astype(np.int8)


@pytest.mark.parametrize("m,n,k", [(1, 3, 128), (5, 7, 256), (16, 33, 384)])
def test_closed_forms_all_zero_plus_minus(m, n, k):
    xq = _xq_random(m, k, 3)
    xs = np.ones(m, dtype=np.float32)
    row_sum = xq.astype(np.int64).sum(axis=1)
    for sign in (0, 1, -1):
        w = np.full((n, k), float(sign), dtype=np.float32)
        _, acc = oracle.gemm(oracle.pack(w), n, k, xq, xs)
        want = np.repeat((sign * row_sum)[:, None], n, axis=1)
        assert np.array_equal(acc.astype(np.int64), want)


@pytest.mark.parametrize("k", [128, 256])
def test_identity_weights_return_the_activations(k):
    xq = _xq_random(4, k, 5)
    _, acc = oracle.gemm(oracle.pack(np.eye(k, dtype=np.float32)), k, k, xq,
                         np.ones(4, dtype=np.float32))
    assert np.array_equal(acc, xq.astype(np.int32))


def test_one_hot_rows_gather_a_permutation():
    k = 256
    perm = np.random.default_rng(9).permutation(k)
    w = np.zeros((k, k), dtype=np.float32)
    w[np.arange(k), perm] = 1.0
    w[::3] *= -1.0  # every third row subtracts
    xq = _xq_random(3, k, 6)
    _, acc = oracle.gemm(oracle.pack(w), k, k, xq, np.ones(3, dtype=np.float32))
    want = xq[:, perm].astype(np.int32)
    want[:, ::3] *= -1
    assert np.array_equal(acc, want)


@pytest.mark.parametrize("n", [1, 2, 3, 7, 33])
@pytest.mark.parametrize("k", [128, 256, 384])
@pytest.mark.parametrize("m", [1, 2, 3, 5, 16])
def test_brute_force_against_integer_matmul(m, n, k):
    w, t, s = inputs.ternary_weights(n, k, 100 * n + k + m)
    xq = _xq_random(m, k, m + 7 * n)
    _, acc = oracle.gemm(oracle.pack(w.numpy()), n, k, xq, np.ones(m, dtype=np.float32))
    want = xq.astype(np.int64) @ t.numpy().astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), want)


def test_int32_range_at_the_longest_reduction():
    k = 28672
    xq = np.full((1, k), 127, dtype=np.int8)
    for sign in (1, -1):
        _, acc = oracle.gemm(oracle.pack(np.full((1, k), float(sign), np.float32)), 1, k, xq,
                             np.ones(1, dtype=np.float32))
        assert int(acc[0, 0]) == sign * 127 * k == sign * 3_641_344


def test_contraction_worked_example():
    ex = _load("contraction_worked_example.json")
    pk = _load("i2s_pack_worked_examples.json")["examples"][1]
    packed = np.frombuffer(bytes.fromhex(pk["expected_hex"]), dtype=np.uint8)
    xq = (np.arange(128) - 64).astype(np.int8)[None, :]
    y, acc = oracle.gemm(packed, 2, 128, xq, np.array(ex["xs"], dtype=np.float32))
    assert acc.tolist() == ex["acc"]
    assert y.tolist() == ex["y"]


def test_dequant_is_within_two_roundings_of_exact_product():
    n, k, m = 17, 256, 6
    w, t, s = inputs.ternary_weights(n, k, 42)
    xq = _xq_random(m, k, 8)
    xs = np.random.default_rng(4).uniform(0.001, 0.2, size=m).astype(np.float32)
    y, acc = oracle.gemm(oracle.pack(w.numpy()), n, k, xq, xs)
    exact = acc.astype(np.float64) * xs.astype(np.float64)[:, None] * float(np.float32(s))
    # two fp32 roundings, each at most half an ulp: relative error <= 2^-23
    err = np.abs(y.astype(np.float64) - exact)
    assert np.all(err <= np.abs(exact) * 2.0 ** -23 + 1e-30)
    assert np.all((y == 0) == (acc == 0))


def test_sampled_outputs_equal_full_outputs():
    n, k, m = 40, 384, 7
    w, _, _ = inputs.ternary_weights(n, k, 77)
    packed = oracle.pack(w.numpy())
    xq, xs = oracle.act_quant(inputs.activations(m, k, 77).numpy())
    y, acc = oracle.gemm(packed, n, k, xq, xs)
    rng = np.random.default_rng(1)
    pm, pn = rng.integers(0, m, 50), rng.integers(0, n, 50)
    ys, accs = oracle.gemm_sampled(packed, n, k, xq, xs, pm, pn)
    assert np.array_equal(accs, acc[pm, pn]) and np.array_equal(ys, y[pm, pn])


# --- activation quantization ---------------------------------------------------

def test_act_quant_worked_examples():
    for ex in _load("act_quant_worked_examples.json")["examples"]:
        xq, xs = oracle.act_quant(np.array(ex["x"], dtype=np.float32))
        assert xq.tolist() == ex["xq"]
        assert xs.tolist() == ex["xs"]


def test_act_quant_error_bound_and_range():
    x = inputs.activations(8, 2560, 5, outliers=True).numpy()
    xq, xs = oracle.act_quant(x)
    assert np.all(np.abs(xq.astype(np.int32)) <= 127)
    amax = np.max(np.abs(x), axis=1)
    # the element of largest magnitude maps to +-127 exactly
    arg = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(xq[np.arange(8), arg].astype(np.int32)) == 127)
    assert np.allclose(xs, amax / 127.0, rtol=2 ** -23)
    # rounding to nearest: |x - xq*xs| <= xs/2, up to the fp32 roundings involved
    err = np.abs(x.astype(np.float64) - xq.astype(np.float64) * xs.astype(np.float64)[:, None])
    assert np.all(err <= xs.astype(np.float64)[:, None] * (0.5 + 1e-5))


def test_act_quant_is_invariant_to_power_of_two_scaling():
    x = inputs.activations(3, 512, 6).numpy()
    xq, xs = oracle.act_quant(x)
    for e in (-3, 4):
        xq2, xs2 = oracle.act_quant(x * np.float32(2.0 ** e))
        assert np.array_equal(xq, xq2)
        assert np.array_equal(xs2, xs * np.float32(2.0 ** e))


def test_act_quant_one_hot_and_zero_rows():
    x = np.zeros((2, 256), dtype=np.float32)
    x[0, 77] = -3.25
    xq, xs = oracle.act_quant(x)
    assert xq[0, 77] == -127 and np.count_nonzero(xq[0]) == 1
    assert not xq[1].any() and xs[1] == 0.0


def test_quant_gemm_is_act_quant_then_gemm():
    n, k, m = 19, 256, 3
    w, _, _ = inputs.ternary_weights(n, k, 8)
    packed = oracle.pack(w.numpy())
    x = inputs.activations(m, k, 8).numpy()
    y, acc, xq, xs = oracle.quant_gemm(packed, n, k, x)
    xq2, xs2 = oracle.act_quant(x)
    y2, acc2 = oracle.gemm(packed, n, k, xq2, xs2)
    assert np.array_equal(xq, xq2) and np.array_equal(acc, acc2) and np.array_equal(y, y2)


# --- AbsMean ternarization and dequantization (next steps) --------------------

def test_absmean_worked_example_keeps_eps_in_the_denominator():
    # "LLM Quantization Paradigms ..." section 5, The Mathematics of BitNet b1.58:
    # gamma = mean|W| = 16/8 = 2; W/(gamma+eps) = [2,-2,~0.5-,~-0.5+,1.5,0,0,1.5];
    # the eps pushes +-0.5 just below one half, so they round to 0.
    w = np.array([4, -4, 1, -1, 3, 0, 0, 3], dtype=np.float32)
    out, gamma = oracle.ternarize_absmean(w, eps=1e-5)
    assert gamma == 2.0
    assert out.tolist() == [2.0, -2.0, 0.0, 0.0, 2.0, 0.0, 0.0, 2.0]


def test_absmean_of_constant_magnitude_is_the_sign():
    w = np.array([0.3, -0.3, 0.3, 0.3, -0.3, -0.3], dtype=np.float32)
    out, gamma = oracle.ternarize_absmean(w, eps=0.0)
    assert np.float32(gamma) == np.float32(0.3)
    assert np.array_equal(np.sign(out), np.sign(w))


def test_absmean_output_packs_losslessly():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((6, 256)).astype(np.float32) * 0.02
    out, gamma = oracle.ternarize_absmean(w)
    t, s = oracle.unpack(oracle.pack(out), 6, 256)
    assert s == np.float32(gamma)
    assert np.array_equal(t.astype(np.float32) * s, out)


def test_dequant_f32_is_codes_times_scale():
    w, t, s = inputs.ternary_weights(9, 384, 12)
    out = oracle.dequant_f32(oracle.pack(w.numpy()), 9, 384)
    assert np.array_equal(out, t.numpy().astype(np.float32) * np.float32(s))


def test_dequant_order_acc_times_token_scale_first():
    # The reading fixes y = ((float)acc * xs) * s.  For these values the other
    # association, acc * (xs * s), rounds differently (194440.921875).  The
    # expected value uses float64 products, which are exact here (22-bit x
    # 24-bit and 24-bit x 24-bit), each rounded once to fp32.
    k = 20224
    acc_target = 2553486
    xs = np.float32(np.uint32(1040900328).view(np.float32))
    s = np.float32(np.uint32(1057995740).view(np.float32))
    xq = np.zeros((1, k), dtype=np.int8)
    xq[0, :20106] = 127
    xq[0, 20106] = acc_target - 127 * 20106
    w = np.full((1, k), s, dtype=np.float32)
    y, acc = oracle.gemm(oracle.pack(w), 1, k, xq, np.array([xs], dtype=np.float32))
    assert int(acc[0, 0]) == acc_target
    step1 = np.float32(float(acc_target) * float(xs))
    step2 = np.float32(float(step1) * float(s))
    assert y[0, 0] == step2 == np.float32(194440.9375)
