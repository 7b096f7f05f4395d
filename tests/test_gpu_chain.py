"""GPU parity of the dependency chain (bitnet_i2s_quant_gemv_chain) against
the oracle's chain, which runs quant_gemm problem by problem on the fp32
outputs it has produced itself.  int32 accumulators must be bit-exact and
fp32 outputs within 1e-5 relative error (tests/parity.py); the chain must
also equal, bit for bit, the same problems run stage by stage through the
batched call.  Shapes span several row tiles, ragged N on the problems no
one reads, K slices (including K > 8192, which needs several), a chain
longer than one launch holds, external inputs in the middle of a chain,
repeats on one workspace and a CUDA graph replay.
"""
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


def _weights(n, k, seed):
    """Seeded ternary weights with a per-tensor scale near 1/sqrt(K/2), so
    values keep their size along a chain."""
    w, t, _ = inputs.ternary_weights(n, k, seed)
    s = np.float32((k / 2) ** -0.5)
    return (t.to(torch.float32) * s), t


class Chain:
    """A chain built from (name, N, K, src) specs, src = index of an earlier
    spec or "x" for an external input of that K.  Keeps host weights for the
    oracle and device tensors for the library; outputs sit in guard bands."""

    def __init__(self, i2s, specs, stages, m, seed, acc=True):
        self.m, self.specs, self.stages = m, specs, stages
        self.w_host, self.packed, self.y, self.acc, self.bufs, self.x = [], [], [], [], [], {}
        for i, (name, n, k, src) in enumerate(specs):
            w, _ = _weights(n, k, seed + 31 * i)
            self.w_host.append(w.numpy())
            self.packed.append(i2s.bitnet_i2s_pack(w.cuda()))
            y, yb = guarded_empty((m, n), torch.float32)
            y.fill_(float("nan"))
            self.y.append(y)
            self.bufs.append(yb)
            if acc:
                a, ab = guarded_empty((m, n), torch.int32)
                self.acc.append(a)
                self.bufs.append(ab)
            else:
                self.acc.append(None)
            if src == "x":
                self.x[i] = inputs.activations(m, k, seed + 17 * i)
        self.x_dev = {i: x.cuda() for i, x in self.x.items()}

    def problems(self):
        out = []
        for i, (name, n, k, src) in enumerate(self.specs):
            x = self.x_dev[i] if src == "x" else self.y[src]
            out.append((self.packed[i], n, k, x, self.y[i], self.acc[i]))
        return out

    def oracle(self):
        probs = []
        for i, (name, n, k, src) in enumerate(self.specs):
            probs.append((oracle.pack(self.w_host[i]), n, k,
                          self.x[i].numpy() if src == "x" else src))
        return oracle.quant_gemm_chain(probs)

    def check(self, ref, what=""):
        torch.cuda.synchronize()
        for i, (y_ref, acc_ref, _, _) in enumerate(ref):
            name = self.specs[i][0]
            assert_y_close(self.y[i].cpu().numpy(), y_ref, f"{what} {i}:{name}")
            if self.acc[i] is not None:
                assert_acc_equal(self.acc[i].cpu().numpy(), acc_ref, f"{what} {i}:{name}")
        assert all(guards_intact(b) for b in self.bufs), what


def layer_specs(layers, hidden, kv, ffn, first_src="x"):
    """Specs and stages of `layers` decoder layers' seven projections."""
    specs, stages = [], []
    h = first_src
    for layer in range(layers):
        base = len(specs)
        st = 4 * layer
        specs += [("q", hidden, hidden, h), ("k", kv, hidden, h), ("v", kv, hidden, h)]
        stages += [st] * 3
        specs.append(("o", hidden, hidden, base))
        stages.append(st + 1)
        specs += [("gate", ffn, hidden, base + 3), ("up", ffn, hidden, base + 3)]
        stages += [st + 2] * 2
        specs.append(("down", hidden, ffn, base + 4))
        stages.append(st + 3)
        h = base + 6
    return specs, stages


@pytest.mark.parametrize("m", [1, 2])
@pytest.mark.parametrize("dims", [(256, 100, 640), (384, 128, 1280), (512, 77, 9216)],
                         ids=["small", "mid", "longK"])
def test_layers_match_the_oracle_chain(i2s, m, dims):
    """Two decoder layers; k and v have ragged N (no one reads them), and the
    longK case's down projection has K = 9216 > 8192 (several slices)."""
    hidden, kv, ffn = dims
    specs, stages = layer_specs(2, hidden, kv, ffn)
    ch = Chain(i2s, specs, stages, m, 900 + hidden)
    i2s.bitnet_i2s_quant_gemv_chain(ch.problems(), stages, m)
    ch.check(ch.oracle(), f"{dims} M={m}")


@pytest.mark.parametrize("m", [1, 2])
def test_chain_equals_stage_by_stage_calls(i2s, m):
    specs, stages = layer_specs(3, 256, 128, 768)
    ch = Chain(i2s, specs, stages, m, 1300)
    probs = ch.problems()
    for st in range(stages[-1] + 1):
        i2s.bitnet_i2s_quant_gemv_batched([p for p, s in zip(probs, stages) if s == st], m)
    torch.cuda.synchronize()
    want_y = [y.clone() for y in ch.y]
    want_acc = [a.clone() for a in ch.acc]
    for y in ch.y:
        y.fill_(float("nan"))
    i2s.bitnet_i2s_quant_gemv_chain(probs, stages, m)
    torch.cuda.synchronize()
    for i in range(len(specs)):
        assert torch.equal(ch.y[i], want_y[i]), i
        assert torch.equal(ch.acc[i], want_acc[i]), i


def test_external_inputs_in_the_middle_and_y_only(i2s):
    """A stage can mix chained and external inputs; problems without an
    accumulator output still feed the next stage."""
    specs = [("a", 256, 384, "x"), ("b", 384, 256, 0), ("c", 384, 256, "x"),
             ("d", 200, 384, 1), ("e", 128, 384, 2), ("f", 256, 128, 4)]
    stages = [0, 1, 1, 2, 2, 3]
    ch = Chain(i2s, specs, stages, 1, 2100, acc=False)
    i2s.bitnet_i2s_quant_gemv_chain(ch.problems(), stages, 1)
    ch.check(ch.oracle(), "mixed")


def test_chain_longer_than_one_launch(i2s):
    """140 problems of one stage each (two launches of up to 128): the second
    launch reads outputs the first wrote."""
    n = 140
    specs = [("p", 128, 128, "x" if i == 0 else i - 1) for i in range(n)]
    stages = list(range(n))
    ch = Chain(i2s, specs, stages, 2, 3100)
    i2s.bitnet_i2s_quant_gemv_chain(ch.problems(), stages, 2)
    ch.check(ch.oracle(), "140 stages")


@pytest.mark.parametrize("m", [1, 2])
def test_one_problem_and_wide_stage(i2s, m):
    """A chain of one problem is the fused call; a stage wider than the grid
    (more row tiles than CTAs) keeps one slice per problem, and the next
    problem reads a 64000-wide row (more than 32 of each warp's 512-chunks,
    so the two-token path polls them in several rounds)."""
    ch = Chain(i2s, [("one", 300, 640, "x")], [0], m, 4100)
    i2s.bitnet_i2s_quant_gemv_chain(ch.problems(), [0], m)
    ch.check(ch.oracle(), "one")
    specs = [("wide", 128 * 500, 256, "x"), ("next", 256, 128 * 500, 0)]
    ch = Chain(i2s, specs, [0, 1], m, 4200)
    i2s.bitnet_i2s_quant_gemv_chain(ch.problems(), [0, 1], m)
    ch.check(ch.oracle(), "wide")


@pytest.mark.parametrize("m", [1, 2])
def test_stage_wider_than_the_grid_reads_chained_sources(i2s, m):
    """Stage 1 has 1000 items (two 64000-row problems), more than the grid's
    CTAs, so CTAs take several of its items and reuse the absmax of a source
    they have already read: b's items (4 boxes each) read their slice again,
    b2's (one box) keep it from the first pass."""
    specs = [("a", 2048, 384, "x"), ("a2", 256, 384, "x"),
             ("b", 128 * 500, 2048, 0), ("b2", 128 * 500, 256, 1)]
    stages = [0, 0, 1, 1]
    ch = Chain(i2s, specs, stages, m, 4300, acc=False)
    i2s.bitnet_i2s_quant_gemv_chain(ch.problems(), stages, m)
    ch.check(ch.oracle(), f"wide stage M={m}")


def test_repeats_on_one_workspace_and_graph_replay(i2s):
    specs, stages = layer_specs(2, 256, 128, 512)
    ch = Chain(i2s, specs, stages, 1, 5100)
    call = i2s.QuantGemvChain(ch.problems(), stages, 1)
    ref = ch.oracle()
    for _ in range(3):
        for y in ch.y:
            y.fill_(float("nan"))
        call.run()
        ch.check(ref, "repeat")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call.run()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call.run()
    for _ in range(3):
        for y in ch.y:
            y.fill_(float("nan"))
        g.replay()
        ch.check(ref, "graph")
    i2s.bitnet_device_status()  # raises if a device-side wait ran out


@pytest.mark.parametrize("m", [1, 2])
def test_staged_stack_as_benchmarked(i2s, m):
    """The benchmark's 30-layer staged step (device-drawn weights): the chain
    equals the 120 stage-by-stage calls bit for bit, and the first two
    layers equal the oracle's chain on the same weights (copied to the host
    and packed by the oracle)."""
    import bench
    staged = bench.staged_problems(i2s, torch, inputs, inputs.LAYERS_2B, m)
    probs, stages = staged[0], staged[1]
    calls, _, _ = bench.staged_stack(i2s, torch, inputs, inputs.LAYERS_2B, m, staged)
    chain, _, _ = bench.staged_chain(i2s, torch, inputs, inputs.LAYERS_2B, m, staged)
    for c in calls:
        c.run()
    torch.cuda.synchronize()
    want = [p[4].clone() for p in probs]
    for p in probs:
        p[4].fill_(float("nan"))
    chain.run()
    torch.cuda.synchronize()
    for i, p in enumerate(probs):
        assert torch.equal(p[4], want[i]), i
    # the oracle on the first two layers (14 problems)
    P = {p.name: p for p in inputs.projections_2b()}
    names = ["q", "k", "v", "o", "gate", "up", "down"]
    srcs = [None, None, None, 0, 3, 3, 4]
    x0 = probs[0][3].cpu().numpy()
    oprobs = []
    for layer in range(2):
        for idx, name in enumerate(names):
            p = P[name]
            w = bench.gpu_ternary(torch, p.n, p.k, inputs.seed_stack(layer, idx),
                                  scale=float((p.k / 2) ** -0.5)).cpu().numpy()
            if srcs[idx] is None:
                src = x0 if layer == 0 else 7 * layer - 1
            else:
                src = 7 * layer + srcs[idx]
            oprobs.append((oracle.pack(w), p.n, p.k, src))
    ref = oracle.quant_gemm_chain(oprobs)
    for i, (y_ref, _, _, _) in enumerate(ref):
        assert_y_close(probs[i][4].cpu().numpy(), y_ref, f"staged {i}")
    assert np.isfinite(probs[-1][4].cpu().numpy()).all()
