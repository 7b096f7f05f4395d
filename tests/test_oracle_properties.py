"""Algebraic properties of the oracle's ternary contraction, on random shapes.

Each property holds for the plain definition acc[m,n] = sum_k w[n,k] xq[m,k]
and fails for the usual indexing slips: a row or column permutation of the
operands must permute or leave the result as the mathematics says, the
contraction is additive over weights with disjoint supports, and it is odd
in the activations.  Inputs are drawn by hypothesis (bounded example counts,
so the CPU suite stays fast); every packed tensor comes from the oracle's own
pack of a known ternary matrix.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle


def _ternary(rng, n, k, p_zero=0.5):
    u = rng.random((n, k))
    w = np.where(u < (1 - p_zero) / 2, -1.0, np.where(u < 1 - (1 - p_zero) / 2, 0.0, 1.0))
    return w.astype(np.float32)


def _acc(w, xq):
    n, k = w.shape
    xs = np.ones(xq.shape[0], dtype=np.float32)
    _, acc = oracle.gemm(oracle.pack(w), n, k, xq, xs)
    return acc.astype(np.int64)


shapes = st.tuples(st.integers(1, 6), st.integers(1, 24), st.sampled_from([128, 256, 384, 512]),
                   st.integers(0, 2**31 - 1))


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_row_permutation_of_weights_permutes_outputs(args):
    m, n, k, seed = args
    rng = np.random.default_rng(seed)
    w = _ternary(rng, n, k)
    xq = rng.integers(-127, 128, (m, k), dtype=np.int8)
    perm = rng.permutation(n)
    np.testing.assert_array_equal(_acc(w[perm], xq), _acc(w, xq)[:, perm])


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_common_column_permutation_leaves_outputs_unchanged(args):
    m, n, k, seed = args
    rng = np.random.default_rng(seed)
    w = _ternary(rng, n, k)
    xq = rng.integers(-127, 128, (m, k), dtype=np.int8)
    perm = rng.permutation(k)  # mixes weights across blocks and groups
    np.testing.assert_array_equal(_acc(w[:, perm], xq[:, perm]), _acc(w, xq))


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_additive_over_weights_with_disjoint_supports(args):
    m, n, k, seed = args
    rng = np.random.default_rng(seed)
    w = _ternary(rng, n, k, p_zero=0.2)
    mask = rng.random((n, k)) < 0.5
    w1 = np.where(mask, w, 0).astype(np.float32)
    w2 = np.where(mask, 0, w).astype(np.float32)
    xq = rng.integers(-127, 128, (m, k), dtype=np.int8)
    # Each part is packed with its own scale (1, or 0 when empty), which the
    # integer accumulators do not see.
    np.testing.assert_array_equal(_acc(w1, xq) + _acc(w2, xq), _acc(w, xq))


@settings(max_examples=25, deadline=None)
@given(shapes)
def test_odd_in_the_activations_and_in_the_weights(args):
    m, n, k, seed = args
    rng = np.random.default_rng(seed)
    w = _ternary(rng, n, k)
    xq = rng.integers(-127, 128, (m, k), dtype=np.int8)  # -xq stays in [-127, 127]
    base = _acc(w, xq)
    np.testing.assert_array_equal(_acc(w, -xq), -base)
    np.testing.assert_array_equal(_acc(-w, xq), -base)
