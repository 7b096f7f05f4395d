"""Seeded synthetic inputs for the I2_S matmul workloads.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no packing, quantization or contraction), so the CUDA
path and the CPU oracle can both be fed from it without sharing any of the
computation under test.  Everything is drawn on the host with a
``torch.Generator`` so both sides see identical bytes.

Shapes are those of BitNet-b1.58-2B-4T as printed in the model metadata on
"ik_llama.cpp 运行 BitNet b1.58 2B 模型实战" (§二, hidden 2560, feed-forward 6912,
30 blocks, 20 query heads and 5 key/value heads of 128), with the seven
ternary projections q, k, v, o, gate, up, down listed on "BitNet Inference
Preprocessing: Converting Hugging Face Checkpoints to I2S GGUF" (Stage 1).

Recipe (stated once here and in the design notes):
  * ternary weights: value -1, 0, +1 with probability 0.25, 0.5, 0.25
    (a uniform draw from {0,1,2,3} mapped 0 -> -1, 1 and 2 -> 0, 3 -> +1),
    times one per-tensor scale s ~ U(0.5, 2);
  * activations: x ~ N(0, 1) fp32; for the "outlier" workload 1% of the K
    channels (chosen once per tensor) are multiplied by 20 for every token,
    the activation-outlier pattern described in "LLM Quantization
    Paradigms: FP8, AWQ, EXL2 & BitNet b1.58 in 2026" §2;
  * seeds: weights use ``seed``, activations ``seed + ACT_SEED_OFFSET``.
"""
from __future__ import annotations

import dataclasses

import torch

ACT_SEED_OFFSET = 1_000_003

HIDDEN_2B = 2560
FFN_2B = 6912
LAYERS_2B = 30
HEAD_DIM = 128
Q_HEADS_2B = 20
KV_HEADS_2B = 5


@dataclasses.dataclass(frozen=True)
class Projection:
    name: str
    n: int  # output rows
    k: int  # input features (reduction length)


def projections_2b() -> list[Projection]:
    """The seven ternary projections of one BitNet-b1.58-2B-4T block."""
    h, f, kv = HIDDEN_2B, FFN_2B, KV_HEADS_2B * HEAD_DIM
    return [
        Projection("q", Q_HEADS_2B * HEAD_DIM, h),
        Projection("k", kv, h),
        Projection("v", kv, h),
        Projection("o", h, Q_HEADS_2B * HEAD_DIM),
        Projection("gate", f, h),
        Projection("up", f, h),
        Projection("down", h, f),
    ]


def projections_large() -> list[Projection]:
    """A larger BitNet-style block: hidden 8192, feed-forward 28672, k/v 1024."""
    h, f, kv = 8192, 28672, 1024
    return [
        Projection("q", h, h),
        Projection("k", kv, h),
        Projection("v", kv, h),
        Projection("o", h, h),
        Projection("gate", f, h),
        Projection("up", f, h),
        Projection("down", h, f),
    ]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def ternary_codes(n: int, k: int, seed: int) -> torch.Tensor:
    """int8 [n, k] with -1 / 0 / +1 drawn with probability 0.25 / 0.5 / 0.25."""
    u = torch.randint(0, 4, (n, k), generator=_gen(seed), dtype=torch.int8)
    t = torch.zeros((n, k), dtype=torch.int8)
    t[u == 0] = -1
    t[u == 3] = 1
    return t


def tensor_scale(seed: int) -> float:
    """The per-tensor scale s ~ U(0.5, 2), as an fp32 value."""
    g = _gen(seed + 7)
    return float(torch.empty(1, dtype=torch.float32).uniform_(0.5, 2.0, generator=g)[0])


def ternary_weights(n: int, k: int, seed: int):
    """(W fp32 [n,k] = T * s, T int8 [n,k], s) for one weight tensor."""
    t = ternary_codes(n, k, seed)
    s = tensor_scale(seed)
    w = t.to(torch.float32) * torch.tensor(s, dtype=torch.float32)
    return w, t, s


def activations(m: int, k: int, seed: int, outliers: bool = False) -> torch.Tensor:
    """fp32 [m, k] ~ N(0,1); with outliers, 1% of channels scaled by 20."""
    g = _gen(seed + ACT_SEED_OFFSET)
    x = torch.randn((m, k), generator=g, dtype=torch.float32)
    if outliers:
        n_out = max(1, round(0.01 * k))
        ch = torch.randperm(k, generator=g)[:n_out]
        x[:, ch] *= 20.0
    return x


# Seeds of the named workloads.
def seed_single() -> int:
    return 0


def seed_layer(proj_index: int) -> int:
    return 1000 + proj_index


def seed_stack(layer: int, proj_index: int) -> int:
    return 10000 + 7 * layer + proj_index


def seed_prefill(shape_index: int) -> int:
    return 20000 + shape_index


def seed_large(proj_index: int) -> int:
    return 30000 + proj_index
