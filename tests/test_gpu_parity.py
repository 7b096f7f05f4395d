"""GPU parity: every C entry point against the CPU oracle on the same seeded inputs.

int32 accumulators and int8/byte outputs must be bit-exact; fp32 outputs
within 1e-5 relative error (tests/parity.py).  Small shapes are compared in
full and span several 128-row tiles, several token tiles and ragged tails in
N, M and K; the workload sizes are compared on sampled outputs (computed one
by one by the oracle) plus an exact whole-output identity.
"""
import numpy as np
import pytest
import torch

import oracle
from i2_mpgemm_b200 import inputs
from tests.parity import (assert_acc_equal, assert_y_close, column_sum_identity, guarded_empty,
                          guards_intact, sample_positions)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def i2s():
    from i2_mpgemm_b200 import i2s as mod
    return mod


def dev(t):
    return t.contiguous().cuda()


# ------------------------------------------------------------------- pack

PACK_SHAPES = [(1, 128), (7, 384), (130, 640), (300, 1152), (640, 2560), (33, 6912)]


@pytest.mark.parametrize("n,k", PACK_SHAPES)
def test_pack_is_byte_exact_on_ternary_weights(i2s, n, k):
    w, _, _ = inputs.ternary_weights(n, k, 5000 + n + k)
    out, buf = guarded_empty((i2s.bitnet_i2s_packed_bytes(n, k),), torch.uint8)
    got = i2s.bitnet_i2s_pack(dev(w), packed=out).cpu().numpy()
    assert np.array_equal(got, oracle.pack(w.numpy()))
    assert guards_intact(buf)


@pytest.mark.parametrize("n,k", PACK_SHAPES[:4])
def test_pack_is_byte_exact_on_arbitrary_weights(i2s, n, k):
    w = torch.randn((n, k), generator=torch.Generator().manual_seed(n * k))
    w[0, 0] = 3.0  # a known maximum; values near +-1.5 exercise the rounding
    w[:, 1] = 1.5
    got = i2s.bitnet_i2s_pack(dev(w)).cpu().numpy()
    assert np.array_equal(got, oracle.pack(w.numpy()))


def test_pack_of_zero_tensor(i2s):
    got = i2s.bitnet_i2s_pack(torch.zeros((3, 256), device="cuda")).cpu().numpy()
    assert np.array_equal(got, oracle.pack(np.zeros((3, 256), np.float32)))


def test_pack_of_every_projection_shape(i2s):
    for idx, p in enumerate(inputs.projections_2b()):
        w, _, _ = inputs.ternary_weights(p.n, p.k, inputs.seed_layer(idx))
        got = i2s.bitnet_i2s_pack(dev(w)).cpu().numpy()
        assert np.array_equal(got, oracle.pack(w.numpy())), p.name


# -------------------------------------------------------- activation quant

@pytest.mark.parametrize("m,k,outliers", [(1, 2560, False), (4, 6912, False), (16, 2560, True),
                                          (37, 384, False), (3, 16, False), (2, 28672, True)])
def test_act_quant_is_bit_exact(i2s, m, k, outliers):
    x = inputs.activations(m, k, 700 + m + k, outliers=outliers)
    xq, xq_buf = guarded_empty((m, k), torch.int8)
    xs, xs_buf = guarded_empty((m,), torch.float32)
    i2s.bitnet_act_quant_i8(dev(x), xq=xq, xs=xs)
    xq_ref, xs_ref = oracle.act_quant(x.numpy())
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(xs.cpu().numpy(), xs_ref)
    assert guards_intact(xq_buf) and guards_intact(xs_buf)


def test_act_quant_worked_examples_and_zero_rows(i2s):
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "act_quant_worked_examples.json")
    for ex in json.load(open(path))["examples"]:
        x = np.zeros((1, 16), np.float32)
        row = np.array(ex["x"][0], np.float32)
        x[0, :row.size] = row  # zero padding leaves amax unchanged
        xq, xs = i2s.bitnet_act_quant_i8(dev(torch.from_numpy(x)))
        assert xq.cpu().numpy()[0, :row.size].tolist() == ex["xq"][0]
        assert xs.cpu().numpy().tolist() == ex["xs"]


# ------------------------------------------------------------- matmul, full

# (M, N, K): several 128-row tiles with ragged N, every token tile size with
# ragged M (past 128 and past 1024 tokens: several 128- or 256-token tiles,
# the last one ragged), and K with a partial last 512-wide stage.
# The tensor-core tile has 127 weight rows (TMEM lane 127 carries the token
# sums), so 127, 128, 254 and 255 rows sit on and next to tile edges; 128 and
# 255 also sit on the decode kernel's.
SMALL = [(1, 1, 128), (1, 7, 640), (3, 130, 384), (16, 300, 1152), (17, 129, 640),
         (33, 257, 512), (64, 200, 1024), (65, 131, 640), (130, 300, 896), (200, 64, 256),
         (5, 127, 256), (9, 124, 384), (20, 128, 384), (70, 254, 640), (3, 255, 128),
         (129, 381, 512), (256, 127, 256), (300, 200, 640), (513, 131, 384),
         (1100, 131, 384), (1025, 254, 640)]


def _case(m, n, k, seed):
    w, t, s = inputs.ternary_weights(n, k, seed)
    x = inputs.activations(m, k, seed, outliers=(seed % 2 == 0))
    packed = oracle.pack(w.numpy())
    xq, xs = oracle.act_quant(x.numpy())
    return w, t, x, packed, xq, xs


@pytest.mark.parametrize("m,n,k", SMALL)
def test_matmul_entries_match_oracle_in_full(i2s, m, n, k):
    w, t, x, packed, xq, xs = _case(m, n, k, 31 * m + n + k)
    y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
    d_packed = dev(torch.from_numpy(packed))
    d_xq, d_xs = dev(torch.from_numpy(xq)), dev(torch.from_numpy(xs))
    entries = [("gemm", i2s.bitnet_i2s_gemm)] + ([("gemv", i2s.bitnet_i2s_gemv)] if m <= 64 else [])
    for name, fn in entries:
        y, y_buf = guarded_empty((m, n), torch.float32)
        acc, acc_buf = guarded_empty((m, n), torch.int32)
        fn(d_packed, n, k, d_xq, d_xs, y=y, acc=acc)
        assert_acc_equal(acc.cpu().numpy(), acc_ref, name)
        assert_y_close(y.cpu().numpy(), y_ref, name)
        assert guards_intact(y_buf) and guards_intact(acc_buf), name
    y, y_buf = guarded_empty((m, n), torch.float32)
    acc, acc_buf = guarded_empty((m, n), torch.int32)
    i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x), y=y, acc=acc)
    assert_acc_equal(acc.cpu().numpy(), acc_ref, "quant_gemv")
    assert_y_close(y.cpu().numpy(), y_ref, "quant_gemv")
    assert guards_intact(y_buf) and guards_intact(acc_buf), "quant_gemv"


def test_y_without_acc_and_repeat_calls_agree(i2s):
    m, n, k = 5, 300, 640
    _, _, x, packed, xq, xs = _case(m, n, k, 9)
    d_packed = dev(torch.from_numpy(packed))
    y1 = i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x))
    y2 = i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x))
    assert torch.equal(y1, y2)
    y_ref, _ = oracle.gemm(packed, n, k, xq, xs)
    assert_y_close(y1.cpu().numpy(), y_ref)


@pytest.mark.parametrize("sign", [1, -1, 0])
@pytest.mark.parametrize("m", [1, 20, 130])
def test_closed_forms_on_gpu(i2s, sign, m):
    n, k = 140, 768
    w = torch.full((n, k), float(sign))
    xq = torch.randint(-127, 128, (m, k), generator=torch.Generator().manual_seed(m),
                       dtype=torch.int8)
    xs = torch.ones(m)
    _, acc = i2s.bitnet_i2s_gemm(i2s.bitnet_i2s_pack(dev(w)), n, k, dev(xq), dev(xs),
                                 want_acc=True)
    want = sign * xq.to(torch.int64).sum(dim=1)
    assert torch.equal(acc.cpu().to(torch.int64), want[:, None].expand(m, n))


def test_identity_weights_on_gpu(i2s):
    k = 256
    xq = torch.randint(-127, 128, (70, k), generator=torch.Generator().manual_seed(2),
                       dtype=torch.int8)
    _, acc = i2s.bitnet_i2s_gemm(i2s.bitnet_i2s_pack(dev(torch.eye(k))), k, k, dev(xq),
                                 dev(torch.ones(70)), want_acc=True)
    assert torch.equal(acc.cpu(), xq.to(torch.int32))


def test_int32_range_at_longest_reduction_on_gpu(i2s):
    k = 28672
    w = torch.ones((3, k))
    w[1] = -1.0
    xq = torch.full((2, k), 127, dtype=torch.int8)
    xq[1] = -127
    _, acc = i2s.bitnet_i2s_gemv(i2s.bitnet_i2s_pack(dev(w)), 3, k, dev(xq), dev(torch.ones(2)),
                                 want_acc=True)
    assert acc.cpu().tolist() == [[3641344, -3641344, 3641344], [-3641344, 3641344, -3641344]]


def test_largest_k(i2s):
    m, n, k = 2, 130, 131072
    _, _, x, packed, xq, xs = _case(m, n, k, 77)
    y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
    y, acc = i2s.bitnet_i2s_quant_gemv(dev(torch.from_numpy(packed)), n, k, dev(x), want_acc=True)
    assert_acc_equal(acc.cpu().numpy(), acc_ref)
    assert_y_close(y.cpu().numpy(), y_ref)


# ---------------------------------------------------- the named workloads

def _packed_pair(i2s, w):
    """(oracle bytes, device bytes) of one weight tensor; the GPU pack must be
    byte-exact.  Oracle inputs always come from the oracle's own pack."""
    packed = oracle.pack(w.numpy())
    d_packed = i2s.bitnet_i2s_pack(dev(w))
    assert np.array_equal(d_packed.cpu().numpy(), packed)
    return packed, d_packed


def _check_full(i2s, packed, d_packed, n, k, x, what):
    y_ref, acc_ref, _, _ = oracle.quant_gemm(packed, n, k, x.numpy())
    y, acc = i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x), want_acc=True)
    assert_acc_equal(acc.cpu().numpy(), acc_ref, what)
    assert_y_close(y.cpu().numpy(), y_ref, what)
    return y, acc


def _check_sampled(i2s, packed, d_packed, n, k, x, t, count, seed, what):
    """quant_gemv at full size: sampled outputs against the oracle, plus the
    exact column-sum identity over every output."""
    m = x.shape[0]
    y, acc = i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x), want_acc=True)
    xq, xs = oracle.act_quant(x.numpy())
    pm, pn = sample_positions(m, n, count, seed)
    y_ref, acc_ref = oracle.gemm_sampled(packed, n, k, xq, xs, pm, pn)
    acc_h, y_h = acc.cpu(), y.cpu()
    assert_acc_equal(acc_h.numpy()[pm, pn], acc_ref, what)
    assert_y_close(y_h.numpy()[pm, pn], y_ref, what)
    assert column_sum_identity(acc_h, torch.from_numpy(xq), t), what


def test_single_k_proj_gemv_in_full(i2s):
    n, k = 640, 2560
    w, t, s = inputs.ternary_weights(n, k, inputs.seed_single())
    x = inputs.activations(1, k, inputs.seed_single())
    packed, d_packed = _packed_pair(i2s, w)
    y, acc = _check_full(i2s, packed, d_packed, n, k, x, "k_proj")
    xq, xs = oracle.act_quant(x.numpy())
    y2, acc2 = i2s.bitnet_i2s_gemv(d_packed, n, k, dev(torch.from_numpy(xq)),
                                   dev(torch.from_numpy(xs)), want_acc=True)
    assert torch.equal(acc2.cpu(), acc.cpu()) and torch.equal(y2.cpu(), y.cpu())


def test_one_layer_decode_with_outliers_in_full(i2s):
    for idx, p in enumerate(inputs.projections_2b()):
        seed = inputs.seed_layer(idx)
        w, t, s = inputs.ternary_weights(p.n, p.k, seed)
        x = inputs.activations(1, p.k, seed, outliers=True)
        packed, d_packed = _packed_pair(i2s, w)
        _check_full(i2s, packed, d_packed, p.n, p.k, x, p.name)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_stack_first_layer_in_full(i2s, m):
    for idx, p in enumerate(inputs.projections_2b()):
        seed = inputs.seed_stack(0, idx)
        w, t, s = inputs.ternary_weights(p.n, p.k, seed)
        x = inputs.activations(m, p.k, seed)
        packed, d_packed = _packed_pair(i2s, w)
        _check_full(i2s, packed, d_packed, p.n, p.k, x, f"{p.name} M={m}")


def test_stack_all_layers_sampled(i2s):
    for layer in range(inputs.LAYERS_2B):
        for idx, p in enumerate(inputs.projections_2b()):
            seed = inputs.seed_stack(layer, idx)
            w, t, s = inputs.ternary_weights(p.n, p.k, seed)
            packed, d_packed = _packed_pair(i2s, w)
            for m in (1, 16):
                x = inputs.activations(m, p.k, seed)
                _check_sampled(i2s, packed, d_packed, p.n, p.k, x, t, 64, seed + m,
                               f"layer {layer} {p.name} M={m}")


@pytest.mark.parametrize("m", [512, 2048])
def test_prefill_shapes_sampled(i2s, m):
    shapes = [("gate", 6912, 2560), ("up", 6912, 2560), ("down", 2560, 6912)]
    for idx, (name, n, k) in enumerate(shapes):
        seed = inputs.seed_prefill(idx)
        w, t, s = inputs.ternary_weights(n, k, seed)
        x = inputs.activations(m, k, seed)
        packed, d_packed = _packed_pair(i2s, w)
        _check_sampled(i2s, packed, d_packed, n, k, x, t, 2048, seed, f"{name} M={m}")


def test_prefill_gate_in_full(i2s):
    """gate 6912x2560 at M = 2048, every output: the int32 accumulators
    against an exact product of the generator's ternary matrix with the
    oracle's int8 codes (float64 BLAS; every sum is below 2^53, so exact),
    and each fp32 output against ((float)acc * xs) * s in that order."""
    n, k, m = 6912, 2560, 2048
    seed = inputs.seed_prefill(0)
    w, t, s = inputs.ternary_weights(n, k, seed)
    x = inputs.activations(m, k, seed)
    packed, d_packed = _packed_pair(i2s, w)
    y, acc = i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x), want_acc=True)
    xq, xs = oracle.act_quant(x.numpy())
    want = (xq.astype(np.float64) @ t.numpy().astype(np.float64).T).astype(np.int64)
    assert_acc_equal(acc.cpu().numpy(), want.astype(np.int32), "gate M=2048")
    scale = np.float32(oracle.scale(packed, n, k))
    y_ref = (want.astype(np.float32) * xs[:, None]).astype(np.float32) * scale
    assert_y_close(y.cpu().numpy(), y_ref.astype(np.float32), "gate M=2048")


@pytest.mark.parametrize("m", [1, 64])
def test_large_layer_sampled(i2s, m):
    for idx, p in enumerate(inputs.projections_large()):
        seed = inputs.seed_large(idx)
        w, t, s = inputs.ternary_weights(p.n, p.k, seed)
        x = inputs.activations(m, p.k, seed)
        packed, d_packed = _packed_pair(i2s, w)
        _check_sampled(i2s, packed, d_packed, p.n, p.k, x, t, 1024, seed + m, f"{p.name} M={m}")
        del d_packed
    torch.cuda.empty_cache()


def test_no_device_wait_timed_out(i2s):
    i2s.bitnet_device_status()


# ------------------------------------------- decode ALU path and batching

# M = 1 with K <= 30720 and M = 2 with K <= 8192 run on the integer-ALU
# decode kernel (K > 8192 on its one-token long-K variant).
# With a workspace (the fused entry) a call with fewer row tiles than CTAs
# splits K across SMs; the pre-quantized entry without one does not, so each
# case checks both.  K = 28672 with 64 and 640 rows: 56 slices of one box.
DECODE = [(1, 1, 128), (1, 300, 2560), (2, 130, 640), (1, 129, 8192), (2, 257, 8192),
          (1, 130, 8320), (1, 257, 28672), (1, 3, 30720),
          (2, 64, 4096), (1, 1000, 6912), (2, 7, 384), (1, 64, 28672), (1, 640, 28672),
          (2, 640, 6912)]


@pytest.mark.parametrize("m,n,k", DECODE)
def test_decode_alu_path_matches_oracle(i2s, m, n, k):
    w, t, x, packed, xq, xs = _case(m, n, k, 17 * m + 3 * n + k)
    y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
    d_packed = dev(torch.from_numpy(packed))
    y, y_buf = guarded_empty((m, n), torch.float32)
    acc, acc_buf = guarded_empty((m, n), torch.int32)
    i2s.bitnet_i2s_gemv(d_packed, n, k, dev(torch.from_numpy(xq)), dev(torch.from_numpy(xs)),
                        y=y, acc=acc)
    assert_acc_equal(acc.cpu().numpy(), acc_ref, "gemv")
    assert_y_close(y.cpu().numpy(), y_ref, "gemv")
    assert guards_intact(y_buf) and guards_intact(acc_buf), "gemv"
    y, y_buf = guarded_empty((m, n), torch.float32)
    acc, acc_buf = guarded_empty((m, n), torch.int32)
    i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x), y=y, acc=acc)
    assert_acc_equal(acc.cpu().numpy(), acc_ref, "quant_gemv")
    assert_y_close(y.cpu().numpy(), y_ref, "quant_gemv")
    assert guards_intact(y_buf) and guards_intact(acc_buf), "quant_gemv"
    # Y alone (no accumulator output), as the benchmark calls it
    y, y_buf = guarded_empty((m, n), torch.float32)
    i2s.bitnet_i2s_quant_gemv(d_packed, n, k, dev(x), y=y)
    assert_y_close(y.cpu().numpy(), y_ref, "quant_gemv, Y only")
    assert guards_intact(y_buf), "quant_gemv, Y only"


def _batched_problems(shapes, m, seed, guards=None):
    """Problems for a batched call; with a `guards` list, every Y and acc is a
    guarded view whose buffer is appended there."""
    cases, problems = [], []
    for i, (n, k) in enumerate(shapes):
        w, t, x, packed, xq, xs = _case(m, n, k, seed + i)
        d_packed, d_x = dev(torch.from_numpy(packed)), dev(x)
        if guards is None:
            y = torch.empty((m, n), device="cuda")
            acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
        else:
            y, yb = guarded_empty((m, n), torch.float32)
            acc, ab = guarded_empty((m, n), torch.int32)
            guards += [yb, ab]
        problems.append((d_packed, n, k, d_x, y, acc))
        cases.append((packed, n, k, xq, xs))
    return cases, problems


@pytest.mark.parametrize("m", [1, 2, 4, 70])
def test_batched_mixed_shapes(i2s, m):
    shapes = [(7, 128), (300, 640), (130, 2560), (64, 6912), (1, 384), (257, 1024)]
    guards = []
    cases, problems = _batched_problems(shapes, m, 900 + m, guards)
    i2s.bitnet_i2s_quant_gemv_batched(problems, m)
    for (packed, n, k, xq, xs), (_, _, _, _, y, acc) in zip(cases, problems):
        y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
        assert_acc_equal(acc.cpu().numpy(), acc_ref, f"{n}x{k}")
        assert_y_close(y.cpu().numpy(), y_ref, f"{n}x{k}")
    assert all(guards_intact(b) for b in guards)


@pytest.mark.parametrize("fused", [True, False], ids=["quant-gemv", "gemv"])
def test_batched_one_token_long_and_short_k(i2s, fused):
    """One token: K <= 8192 and 8192 < K <= 30720 problems go to separate
    launches of the two decode variants within one call."""
    m = 1
    shapes = [(130, 2560), (257, 28672), (7, 128), (33, 12288), (640, 2560), (65, 30720)]
    cases, problems = _batched_problems(shapes, m, 5100)
    if fused:
        i2s.bitnet_i2s_quant_gemv_batched(problems, m)
    else:
        q = []
        for (packed, n, k, xq, xs), (d_packed, _, _, _, y, acc) in zip(cases, problems):
            q.append((d_packed, n, k, dev(torch.from_numpy(xq)), dev(torch.from_numpy(xs)), y, acc))
        i2s.bitnet_i2s_gemv_batched(q, m)
    for (packed, n, k, xq, xs), pr in zip(cases, problems):
        y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
        assert_acc_equal(pr[5].cpu().numpy(), acc_ref, f"{n}x{k}")
        assert_y_close(pr[4].cpu().numpy(), y_ref, f"{n}x{k}")


def test_batched_more_than_one_launch_worth_of_problems(i2s):
    shapes = [(3 + (i % 5), 128 * (1 + i % 3)) for i in range(300)]
    cases, problems = _batched_problems(shapes, 1, 4000)
    plan = i2s.BatchedQuantGemv(problems, 1)
    plan.run()
    plan.run()  # a second call on the same workspace gives the same results
    for (packed, n, k, xq, xs), (_, _, _, _, y, acc) in zip(cases, problems):
        y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
        assert_acc_equal(acc.cpu().numpy(), acc_ref)
        assert_y_close(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("m", [1, 2, 16])
def test_stack_batched_all_layers_sampled(i2s, m):
    """The 210-projection stack through one batched call, as the benchmark runs it."""
    problems, keep = [], []
    for layer in range(inputs.LAYERS_2B):
        for idx, p in enumerate(inputs.projections_2b()):
            seed = inputs.seed_stack(layer, idx)
            w, t, s = inputs.ternary_weights(p.n, p.k, seed)
            x = inputs.activations(m, p.k, seed)
            packed = oracle.pack(w.numpy())
            d_packed = dev(torch.from_numpy(packed))
            y = torch.empty((m, p.n), device="cuda")
            acc = torch.empty((m, p.n), dtype=torch.int32, device="cuda")
            problems.append((d_packed, p.n, p.k, dev(x), y, acc))
            keep.append((packed, p.n, p.k, x, t, seed))
    i2s.bitnet_i2s_quant_gemv_batched(problems, m)
    torch.cuda.synchronize()
    for (packed, n, k, x, t, seed), (_, _, _, _, y, acc) in zip(keep, problems):
        xq, xs = oracle.act_quant(x.numpy())
        pm, pn = sample_positions(m, n, 32, seed)
        y_ref, acc_ref = oracle.gemm_sampled(packed, n, k, xq, xs, pm, pn)
        acc_h = acc.cpu()
        assert_acc_equal(acc_h.numpy()[pm, pn], acc_ref, f"{n}x{k}")
        assert_y_close(y.cpu().numpy()[pm, pn], y_ref, f"{n}x{k}")
        assert column_sum_identity(acc_h, torch.from_numpy(xq), t)


@pytest.mark.parametrize("m", [1, 2])
def test_stack_exactly_as_benchmarked(i2s, m):
    """The benchmark's own step: bench.Stack's 210 problems with Y only (no
    accumulator output), one BatchedQuantGemv call as bench.stack_batch builds
    it.  Y of the whole first layer is compared in full with the oracle, and
    32 sampled outputs plus the corners and the last row tile of every other
    problem; the weights are packed on both sides independently (the oracle's
    pack from the host weights, the library's inside bench.Stack)."""
    import bench
    stack = bench.Stack(i2s, torch, inputs, inputs.LAYERS_2B, m, act_seed_offset=0)
    plan = bench.stack_batch(i2s, stack.probs)
    stack.y_dev.fill_(float("nan"))
    plan.run()
    torch.cuda.synchronize()
    shapes = [(layer, idx, p) for layer in range(inputs.LAYERS_2B)
              for idx, p in enumerate(inputs.projections_2b())]
    assert len(shapes) == len(stack.probs)
    for (layer, idx, p), pr in zip(shapes, stack.probs):
        seed = inputs.seed_stack(layer, idx)
        w, t, s = inputs.ternary_weights(p.n, p.k, seed)
        packed = oracle.pack(w.numpy())
        x = inputs.activations(m, p.k, seed)
        y = pr.y.cpu().numpy()
        what = f"layer {layer} {p.name} M={m}"
        if layer == 0:
            y_ref, _, _, _ = oracle.quant_gemm(packed, p.n, p.k, x.numpy())
            assert_y_close(y, y_ref, what)
        else:
            xq, xs = oracle.act_quant(x.numpy())
            pm, pn = sample_positions(m, p.n, 32, seed)
            y_ref, _ = oracle.gemm_sampled(packed, p.n, p.k, xq, xs, pm, pn)
            assert_y_close(y[pm, pn], y_ref, what)
    assert np.isfinite(stack.y_dev.cpu().numpy()).all()


@pytest.mark.parametrize("workspace", [True, None], ids=["work-counter", "fixed-ranges"])
@pytest.mark.parametrize("m", [1, 2, 5])
def test_gemv_batched_on_quantized_inputs(i2s, m, workspace):
    shapes = [(640, 2560), (640, 2560), (2560, 2560), (33, 6912), (130, 128)]
    cases, problems = [], []
    for i, (n, k) in enumerate(shapes):
        w, t, x, packed, xq, xs = _case(m, n, k, 7000 + i)
        y = torch.empty((m, n), device="cuda")
        acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
        problems.append((dev(torch.from_numpy(packed)), n, k, dev(torch.from_numpy(xq)),
                         dev(torch.from_numpy(xs)), y, acc))
        cases.append((packed, n, k, xq, xs))
    i2s.bitnet_i2s_gemv_batched(problems, m, workspace=workspace)
    for (packed, n, k, xq, xs), pr in zip(cases, problems):
        y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
        assert_acc_equal(pr[6].cpu().numpy(), acc_ref)
        assert_y_close(pr[5].cpu().numpy(), y_ref)


@pytest.mark.parametrize("workspace", [True, None], ids=["work-counter", "fixed-ranges"])
def test_gemv_batched_many_problems_repeated_on_one_workspace(i2s, workspace):
    """Two integer-ALU launches; with a workspace, its counters are zeroed by
    every call, so repeating the call on the same workspace gives the same
    results (every output is poisoned in between)."""
    m = 1
    shapes = [(40 + 97 * (i % 7), 128 * (1 + i % 5)) for i in range(170)]
    cases, problems = [], []
    for i, (n, k) in enumerate(shapes):
        w, t, x, packed, xq, xs = _case(m, n, k, 8000 + i)
        y = torch.empty((m, n), device="cuda")
        acc = torch.empty((m, n), dtype=torch.int32, device="cuda")
        problems.append((dev(torch.from_numpy(packed)), n, k, dev(torch.from_numpy(xq)),
                         dev(torch.from_numpy(xs)), y, acc))
        cases.append((packed, n, k, xq, xs))
    plan = i2s.BatchedGemv(problems, m, workspace=workspace)
    for _ in range(2):
        for pr in problems:
            pr[5].fill_(float("nan"))
            pr[6].fill_(-1)
        plan.run()
        for (packed, n, k, xq, xs), pr in zip(cases, problems):
            y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
            assert_acc_equal(pr[6].cpu().numpy(), acc_ref, f"{n}x{k}")
            assert_y_close(pr[5].cpu().numpy(), y_ref, f"{n}x{k}")


# ------------------------------------------------ dequant and ternarization

@pytest.mark.parametrize("n,k", [(1, 128), (7, 384), (130, 640), (640, 2560), (33, 6912)])
def test_dequant_f32_is_exact(i2s, n, k):
    w, t, s = inputs.ternary_weights(n, k, 8100 + n + k)
    packed = oracle.pack(w.numpy())
    out, buf = guarded_empty((n, k), torch.float32)
    got = i2s.bitnet_i2s_dequant_f32(dev(torch.from_numpy(packed)), n, k, w_out=out).cpu().numpy()
    assert np.array_equal(got, oracle.dequant_f32(packed, n, k))
    assert np.array_equal(got, w.numpy())  # lossless on ternary x scale
    assert guards_intact(buf)


@pytest.mark.parametrize("n,k", [(3, 128), (64, 2560), (640, 2560), (2560, 6912)])
def test_ternarize_absmean_matches_oracle(i2s, n, k):
    g = torch.Generator().manual_seed(n * 7 + k)
    w = torch.randn((n, k), generator=g) * 0.02
    out, buf = guarded_empty((n, k), torch.float32)
    _, gamma = i2s.bitnet_ternarize_absmean(dev(w), eps=1e-5, w_out=out)
    out_ref, gamma_ref = oracle.ternarize_absmean(w.numpy(), eps=1e-5)
    gam = float(gamma.cpu()[0])
    # gamma: the same fp64 sum in another order, so equal up to rounding
    assert abs(gam - gamma_ref) <= 1e-12 * abs(gamma_ref)
    # The codes are decided in fp64 on both sides from gammas that differ by
    # at most that rounding, so they agree unless some |W/(gamma+eps)| lies
    # that close to 1/2.  These inputs have no such element: check it, so
    # that no element is left out of the comparison below.
    t = w.numpy().astype(np.float64) / (gamma_ref + 1e-5)
    assert not np.any(np.abs(np.abs(t) - 0.5) < 1e-9)
    got = out.cpu().numpy()
    assert np.array_equal(np.sign(got), np.sign(out_ref))
    # W_out = code * (float)gamma on both sides: within 1e-5 of the oracle's
    # output (the two (float)gamma differ by at most one rounding), and
    # exactly zero where the oracle's is
    assert_y_close(got, out_ref, "ternarize W_out")
    assert guards_intact(buf)
    # the output packs losslessly with scale (float)gamma
    codes = np.sign(got).astype(np.int8)
    t2, s2 = oracle.unpack(oracle.pack(got), n, k)
    if np.any(codes != 0):
        assert s2 == np.float32(gam)
    assert np.array_equal(t2, codes)


def test_ternarize_worked_example_on_gpu(i2s):
    w = torch.tensor([4, -4, 1, -1, 3, 0, 0, 3], dtype=torch.float32)
    out, gamma = i2s.bitnet_ternarize_absmean(dev(w), eps=1e-5)
    assert float(gamma.cpu()[0]) == 2.0
    assert out.cpu().tolist() == [2.0, -2.0, 0.0, 0.0, 2.0, 0.0, 0.0, 2.0]


def test_batched_tensor_path_over_several_launches(i2s):
    # 4 tokens: every problem goes to the tensor-core kernel, 200 problems
    # span several launches of the persistent kernel.
    shapes = [(3 + 61 * (i % 4), 128 * (1 + i % 5)) for i in range(200)]
    cases, problems = _batched_problems(shapes, 4, 6000)
    i2s.bitnet_i2s_quant_gemv_batched(problems, 4)
    for (packed, n, k, xq, xs), (_, _, _, _, y, acc) in zip(cases, problems):
        y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
        assert_acc_equal(acc.cpu().numpy(), acc_ref, f"{n}x{k}")
        assert_y_close(y.cpu().numpy(), y_ref, f"{n}x{k}")


# ------------------------------------------------------- failure detection

def test_a_device_wait_that_runs_out_is_reported_and_cleared(i2s):
    i2s.bitnet_device_status()  # start clean
    i2s.bitnet_debug_wait_timeout(2_000_000)  # 2 ms, on a barrier nothing completes
    with pytest.raises(i2s.BitnetError) as err:
        i2s.bitnet_device_status()
    assert err.value.status == 5  # BITNET_ERR_DEVICE_TIMEOUT
    i2s.bitnet_device_status()  # the flag was cleared
    # the context is still usable afterwards
    w, _, _ = inputs.ternary_weights(7, 128, 3)
    assert np.array_equal(i2s.bitnet_i2s_pack(dev(w)).cpu().numpy(), oracle.pack(w.numpy()))


@pytest.mark.parametrize("m", [1, 2])
def test_split_k_batches_repeat_on_one_workspace(i2s, m):
    """A qkv-like batch (three problems, 30 row tiles) splits K across SMs;
    calling it twice on the same workspace, with every output poisoned in
    between, gives the oracle's results both times (the arrival counters are
    zeroed by each call)."""
    shapes = [(2560, 2560), (640, 2560), (640, 2560)]
    guards = []
    cases, problems = _batched_problems(shapes, m, 9100 + m, guards)
    plan = i2s.BatchedQuantGemv(problems, m)
    for _ in range(2):
        for pr in problems:
            pr[4].fill_(float("nan"))
            pr[5].fill_(-1)
        plan.run()
        for (packed, n, k, xq, xs), pr in zip(cases, problems):
            y_ref, acc_ref = oracle.gemm(packed, n, k, xq, xs)
            assert_acc_equal(pr[5].cpu().numpy(), acc_ref, f"{n}x{k}")
            assert_y_close(pr[4].cpu().numpy(), y_ref, f"{n}x{k}")
    assert all(guards_intact(b) for b in guards)
