#!/usr/bin/env python
"""Benchmark of the I2_S ternary x int8 matmul on B200.

Default workload (the JSON line's `value`, `--config 2`): one decode step of
the full BitNet-b1.58-2B-4T projection stack -- 30 layers x 7 projections
(q/o 2560x2560, k/v 640x2560, gate/up 6912x2560, down 2560x6912) = 210 fused
activation-quant + ternary matmuls at batch 1, each with its own seeded fp32
input.  The 521 MB of packed weights stay resident in HBM; the working set is
over 4x the 126 MB L2, so every step streams them from HBM.  One step is one
replay of a CUDA graph holding one call of the public C ABI,
bitnet_i2s_quant_gemv_batched, over the 210 problems.  `value` is
packed-weight GB/s over all ranks.

`--config` picks another workload for the line (each streams more than L2
per step, or rotates over distinct copies that together do):
  0  one k_proj GEMV (640x2560, batch 1): 1231 distinct packed copies per
     step in one batched fused call, plus the latency of a single call
  1  one layer's 7 projections at batch 1 with 1 % x20 outlier channels,
     rotated over 16 distinct copies of the layer, one call per step
  2  the 30-layer stack (default), at --batch tokens
  3  prefill GEMM: gate/up 6912x2560 and down 2560x6912 at --batch tokens
     (default 2048) in one fused call per step; value in TOPS
  4  a large BitNet-style layer (hidden 8192, ffn 28672), two copies at
     batch 1 (GB/s), or one copy at --batch 64 (GB/s and TOPS)

Secondary measurements (default run only) land in `extra`: the stack as 210
separate calls; as a dependency-staged decode step (120 ordered calls, each
stage reading the previous stage's output); a sustained run of the headline
step over about a second with its clocks; the stack at batch 2, 4 and 16;
prefill TOPS; the other configs' figures.

Multi-GPU (`--gpus N` under torchrun): every rank holds a replica of the
weights and runs its own token batch (data parallel, weak scaling); there is
no collective on the data path, only a barrier and a max-reduction of the
timings.

`--impl reference` times the CPU oracle (scalar C, one thread) on a bounded
sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "I2_S ternary GEMV/GEMM: packed-weight GB/s & % HBM roofline; prefill TOPS"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_INT8_OVER_BF16 = 2.0  # 4.5 POPS int8 dense / 2.25 PFLOP/s bf16 dense
DECODE_BATCH = 160  # problems per launch of the decode kernel
MMA_BATCH = 96  # problems per launch of the tensor-core kernel
L2_BYTES = 126e6
# (N, K) of the seven projections of one BitNet-b1.58-2B-4T block
STACK_SHAPES = [(2560, 2560), (640, 2560), (640, 2560), (2560, 2560), (6912, 2560), (6912, 2560),
                (2560, 6912)]
TRAFFIC_SUMMARY = os.path.join(ROOT, "profiles", "i2s_gemv_dp4a_stack_batch1.md")
DECODE_SOURCES = [os.path.join(ROOT, "i2_mpgemm_b200", "csrc", f)
                  for f in ("gemv_kernel.cuh", "ptx.cuh")]
DEFAULT_BATCH = {0: 1, 1: 1, 2: 1, 3: 2048, 4: 1}


# ------------------------------------------------------------------ setup

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", type=int, choices=[0, 1, 2, 3, 4], default=2,
                    help="workload (see the module docstring); 2 is the 30-layer stack")
    ap.add_argument("--batch", type=int, default=None,
                    help="tokens per step (default: 1, or 2048 for --config 3)")
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary measurements")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the gate 6912x2560 prefill GEMM at M=2048 (a small case "
                         "for profiling the tensor-core kernel) and print its own line")
    ap.add_argument("--chain-only", action="store_true",
                    help="time only the dependency-staged 30-layer step as one chain call at "
                         "--batch tokens (1 or 2; a case for profiling the chain kernel) and "
                         "print its own line")
    args = ap.parse_args(argv)
    if args.batch is None:
        args.batch = DEFAULT_BATCH[args.config]
    return args


def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 process if absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_init(backend: str):
    import datetime

    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def step_launches(m: int, ks) -> int:
    """Kernel launches of one batched fused call on problems with these K:
    one quantizer launch per 1000 problems, decode launches of up to
    DECODE_BATCH problems (M <= 2 with K <= 8192, or M = 1 with K <= 30720),
    tensor-core launches of up to MMA_BATCH problems for the rest."""
    ks = list(ks)
    small = sum(1 for k in ks if (m <= 2 and k <= 8192) or (m == 1 and k <= 30720))
    return -(-len(ks) // 1000) + -(-small // DECODE_BATCH) + -(-(len(ks) - small) // MMA_BATCH)


def prefill_tile(m: int) -> int:
    """Token tile of the shared-memory tensor kernel at M tokens (the library
    routes 33-64 tokens to 64-token tiles, up to 1024 to 128, above to 256)."""
    return 64 if m <= 64 else (128 if m <= 1024 else 256)


def code_digest(paths) -> str:
    """sha256 of the code of the given sources with comments and blank lines
    removed, so that a comment edit keeps a capture valid and a code edit
    does not."""
    import hashlib
    import re
    parts = []
    for path in paths:
        text = open(path).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        parts.append("\n".join(l.rstrip() for l in text.splitlines() if l.strip()))
    return hashlib.sha256("\n".join(parts).encode()).hexdigest()


def measured_traffic():
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, or None when the kernel's code changed since the capture."""
    try:
        text = open(TRAFFIC_SUMMARY).read()
        src = code_digest(DECODE_SOURCES)
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            key, _, val = line.strip()[2:].partition(":")
            vals[key.strip()] = val.strip().strip("`")
    if vals.get("kernel code sha256") != src:
        return None
    try:
        return int(vals["dram bytes per launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.gpu_id = gpu_id
        self.lines = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def samples(self):
        """[(sm_mhz, max_mhz, power_w, {reasons active})] per sample."""
        out = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            try:
                pw = float(parts[3])
            except ValueError:
                pw = float("nan")
            reasons = {n for n, v in zip(names, parts[5:9]) if v.lower().startswith("active")}
            out.append((sm, mx, pw, reasons))
        return out

    def summary(self):
        s = self.samples()
        if not s:
            return None
        reasons = set()
        for *_, r in s:
            reasons |= r
        return {"sm_mhz": statistics.median(x[0] for x in s), "sm_max_mhz": max(x[1] for x in s),
                "samples": len(s), "reasons": sorted(reasons)}


def gpu_uuid(torch, device_index: int) -> str | None:
    try:
        u = str(torch.cuda.get_device_properties(device_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# ------------------------------------------------------------- workloads

class Problem:
    """One projection: resident packed weights plus views of the step buffers."""

    def __init__(self, i2s, torch, n, k, m, w, x, y, packed=None):
        self.n, self.k, self.m = n, k, m
        self.packed = i2s.bitnet_i2s_pack(w.cuda()) if packed is None else packed
        self.packed_bytes = n * k // 4
        self.x, self.y = x, y
        self.ws = torch.empty(i2s.bitnet_i2s_quant_gemv_workspace_bytes(m, k), dtype=torch.uint8,
                              device="cuda")


class Buffers:
    """Every step input in one device buffer and every output in another
    (each problem's X and Y are views), with pinned host copies, so an
    end-to-end step moves a step's inputs and outputs with one copy each."""

    def __init__(self, torch, x_total: int, y_total: int):
        self.x_dev = torch.empty(x_total, dtype=torch.float32, device="cuda")
        self.y_dev = torch.empty(y_total, dtype=torch.float32, device="cuda")
        self.x_host = torch.empty(x_total, dtype=torch.float32).pin_memory()
        self.y_host = torch.empty(y_total, dtype=torch.float32).pin_memory()
        self.xo = self.yo = 0

    def take(self, m, k, n):
        x = self.x_dev[self.xo:self.xo + m * k].view(m, k)
        y = self.y_dev[self.yo:self.yo + m * n].view(m, n)
        xh = self.x_host[self.xo:self.xo + m * k]
        self.xo += m * k
        self.yo += m * n
        return x, y, xh


class Stack:
    """The projection stack (layers x 7 problems) in one Buffers."""

    def __init__(self, i2s, torch, inputs, layers: int, m: int, act_seed_offset: int,
                 outliers: bool = False, seed_fn=None):
        seed_fn = seed_fn or inputs.seed_stack
        shapes = [(layer, idx, p) for layer in range(layers)
                  for idx, p in enumerate(inputs.projections_2b())]
        self.buf = Buffers(torch, sum(m * p.k for _, _, p in shapes),
                           sum(m * p.n for _, _, p in shapes))
        self.probs = []
        for layer, idx, p in shapes:
            seed = seed_fn(layer, idx)
            w, _, _ = inputs.ternary_weights(p.n, p.k, seed)
            x, y, xh = self.buf.take(m, p.k, p.n)
            xh.copy_(inputs.activations(m, p.k, seed + act_seed_offset, outliers=outliers)
                     .reshape(-1))
            self.probs.append(Problem(i2s, torch, p.n, p.k, m, w, x, y))
            del w
        self.x_dev, self.y_dev = self.buf.x_dev, self.buf.y_dev
        self.x_host, self.y_host = self.buf.x_host, self.buf.y_host
        self.x_dev.copy_(self.x_host)
        torch.cuda.synchronize()

    def h2d(self):
        self.x_dev.copy_(self.x_host, non_blocking=True)

    def d2h(self):
        self.y_host.copy_(self.y_dev, non_blocking=True)


def build_stack(i2s, torch, inputs, layers: int, m: int, act_seed_offset: int):
    return Stack(i2s, torch, inputs, layers, m, act_seed_offset).probs


def stack_step(i2s, probs):
    """The stack as 210 separate fused calls (two launches each)."""
    for pr in probs:
        i2s.bitnet_i2s_quant_gemv(pr.packed, pr.n, pr.k, pr.x, y=pr.y, workspace=pr.ws)


def stack_batch(i2s, probs):
    """The stack as one batched fused call."""
    return i2s.BatchedQuantGemv([(p.packed, p.n, p.k, p.x, p.y, None) for p in probs], probs[0].m)


def capture(torch, fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm: per-device kernel attributes are set outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_replays(torch, g, steps: int, warmup: int, before=None, after=None,
                 collective: bool = True) -> float:
    """Milliseconds per step, CUDA events on the replay stream.  `g` is one
    graph (replayed every step) or a list of graphs (step i replays
    g[i % len(g)]; `before`/`after` then get i).  With `collective`, every
    rank must call it (barriers before and after); rank-0-only measurements
    pass collective=False."""
    graphs = g if isinstance(g, list) else [g]
    rot = isinstance(g, list)

    def one(i):
        if before:
            before(i) if rot else before()
        graphs[i % len(graphs)].replay()
        if after:
            after(i) if rot else after()

    # A graph's first replay uploads it to the device; every graph of a
    # rotation gets that replay here, so no upload lands in the timed region.
    if rot:
        for i in range(len(graphs)):
            one(i)
    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    if collective:
        barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        one(i)
    end.record()
    end.synchronize()
    torch.cuda.synchronize()
    if collective:
        barrier()
    return start.elapsed_time(end) / steps


def matmul_kernel_time(i2s, torch, plans_probs, reps: int = 20):
    """Average device time of the matmul launch(es) of one step, CUDA events
    on the launching stream, with the activations quantized beforehand so the
    timed region holds only the matmul kernels (and, for the decode kernel,
    the one-warp reset of its work counters).  `plans_probs` is a list of
    steps, each a list of Problem; the timed loop rotates over them.
    Returns (ms per step, launches per step, algorithmic bytes per step)."""
    plans, nbytes = [], 0
    for probs in plans_probs:
        qs = [i2s.bitnet_act_quant_i8(p.x) for p in probs]
        m = probs[0].m
        plans.append(i2s.BatchedGemv([(p.packed, p.n, p.k, q, s, p.y, None)
                                      for p, (q, s) in zip(probs, qs)], m))
        nbytes += sum(p.packed_bytes + 4 + p.m * p.k + 4 * p.m + 4 * p.m * p.n for p in probs)
    probs = plans_probs[0]
    m = probs[0].m
    small = [p for p in probs if (m <= 2 and p.k <= 8192) or (m == 1 and p.k <= 30720)]
    launches = -(-len(small) // DECODE_BATCH) + -(-(len(probs) - len(small)) // MMA_BATCH)
    for _ in range(3):
        for pl in plans:
            pl.run()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(reps * len(plans)):
        plans[i % len(plans)].run()
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / (reps * len(plans))
    return ms, launches, nbytes / len(plans)


# ------------------------------------------------------------ CPU oracle

def oracle_layer_sample(inputs, m: int, outliers: bool = False, seed_fn=None):
    """One layer's seven projections packed by the oracle, with inputs."""
    import oracle
    seed_fn = seed_fn or inputs.seed_stack
    sample = []
    for idx, p in enumerate(inputs.projections_2b()):
        seed = seed_fn(0, idx)
        w, _, _ = inputs.ternary_weights(p.n, p.k, seed)
        x = inputs.activations(m, p.k, seed, outliers=outliers)
        sample.append((oracle.pack(w.numpy()), p.n, p.k, x.numpy()))
    return sample


def oracle_sample(inputs, config: int, m: int, w_large=None):
    """The bounded sample of a config's workload that the oracle runs: a list
    of (packed, n, k, x) problems, the unit of the rate, the work per pass
    in that unit's base (bytes or int ops), and a description.  For config 4
    `w_large` is the down projection's fp32 ternary weights as the timed arm
    drew them (seeded torch RNG on the device, copied to the host); the oracle
    packs them itself.  Without it the host generator draws weights of the
    same shape and distribution (timing only)."""
    import oracle
    if config == 0:
        w, _, _ = inputs.ternary_weights(640, 2560, inputs.seed_single())
        x = inputs.activations(m, 2560, inputs.seed_single())
        s = [(oracle.pack(w.numpy()), 640, 2560, x.numpy())]
        return s, "GB/s", 640 * 2560 // 4, f"the k_proj 640x2560 GEMV at batch {m}"
    if config in (1, 2):
        outl = config == 1
        seed_fn = (lambda layer, idx: inputs.seed_layer(idx)) if outl else None
        s = oracle_layer_sample(inputs, m, outliers=outl, seed_fn=seed_fn)
        what = ("the layer's 7 projections with outliers" if outl else
                "one layer's 7 projections (1/30 of the stack)")
        return s, "GB/s", sum(n * k // 4 for _, n, k, _ in s), f"{what} at batch {m}"
    if config == 3:
        tok = min(m, 4)  # a few of the prompt's tokens through gate, up and down
        s = []
        for idx, (n, k) in enumerate([(6912, 2560), (6912, 2560), (2560, 6912)]):
            seed = inputs.seed_prefill(idx)
            w, _, _ = inputs.ternary_weights(n, k, seed)
            x = inputs.activations(m, k, seed)[:tok]
            s.append((oracle.pack(w.numpy()), n, k, x.numpy()))
        return s, "TOPS", sum(2 * tok * n * k for _, n, k, _ in s), \
            f"the first {tok} of the {m} tokens through gate, up and down"
    p = inputs.projections_large()[6]  # down 8192 x 28672
    w = w_large if w_large is not None else inputs.ternary_weights(p.n, p.k, inputs.seed_large(6))[0]
    x = inputs.activations(1, p.k, inputs.seed_large(6))
    return [(oracle.pack(w.numpy()), p.n, p.k, x.numpy())], "GB/s", p.n * p.k // 4, \
        "the large layer's down projection 8192x28672 at batch 1"


def oracle_pass(sample):
    """One pass of the oracle over a sample: (seconds, outputs)."""
    import oracle
    t0 = time.perf_counter()
    ys = [oracle.quant_gemm(packed, n, k, x)[0] for packed, n, k, x in sample]
    return time.perf_counter() - t0, ys


def rate(work: float, seconds: float, unit: str) -> float:
    return work / seconds / (1e9 if unit == "GB/s" else 1e12)


def cpu_baseline(inputs, config: int, m: int, budget_s: float, gpu_outputs=None, w_large=None):
    """The oracle, one thread, on the config's bounded sample for about
    `budget_s`.  With `gpu_outputs` (the timed step's outputs of the same
    sample problems, host arrays), the first pass's outputs are compared
    with them at the tests' tolerance, and the verdict is reported."""
    sample, unit, work, what = oracle_sample(inputs, config, m, w_large)
    done, spent, ys = 0, 0.0, None
    while spent < budget_s or done == 0:
        dt, out = oracle_pass(sample)
        ys = ys or out
        spent += dt
        done += 1
    res = {"value": round(rate(done * work, spent, unit), 6), "unit": unit, "cores": 1,
           "kind": "oracle",
           "sample": f"{done} passes over {what} (scalar C oracle, one thread, {spent:.1f} s)"}
    if gpu_outputs is not None:
        res["parity"] = compare_outputs(gpu_outputs, ys)
    return res


def compare_outputs(got, want):
    """Element-wise comparison of the GPU step's outputs with the oracle's:
    within 1e-5 relative error and exactly zero where the oracle's is."""
    import numpy as np
    worst, count, ok = 0.0, 0, True
    for g, w in zip(got, want):
        g = np.asarray(g, dtype=np.float64).reshape(w.shape)
        w = np.asarray(w, dtype=np.float64)
        zero = w == 0
        ok = ok and bool(np.all(g[zero] == 0))
        if (~zero).any():
            worst = max(worst, float(np.max(np.abs(g[~zero] - w[~zero]) / np.abs(w[~zero]))))
        count += w.size
    ok = ok and worst <= 1e-5
    return {"parity_ok": ok, "outputs_compared": count, "max_rel_err": worst}


_WORKER_SAMPLE = None


def _oracle_worker_init(m: int):
    global _WORKER_SAMPLE
    from i2_mpgemm_b200 import inputs
    _WORKER_SAMPLE = oracle_layer_sample(inputs, m)


def _oracle_worker_task(idx: int) -> int:
    import oracle
    packed, n, k, x = _WORKER_SAMPLE[idx]
    oracle.quant_gemm(packed, n, k, x)
    return n * k // 4


def cpu_baseline_all_cores(m: int, budget_s: float):
    """The same oracle, one process per host core (spawned: the parent has a
    CUDA context), each taking whole projections of the one-layer sample."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    cores = os.cpu_count() or 1
    # A worker that dies raises here instead of being replaced forever.
    with ProcessPoolExecutor(cores, mp_context=mp.get_context("spawn"),
                             initializer=_oracle_worker_init, initargs=(m,)) as pool:
        list(pool.map(_oracle_worker_task, list(range(7)) * cores))  # warm every worker
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < budget_s:
            done += sum(pool.map(_oracle_worker_task, list(range(7)) * cores))
        spent = time.perf_counter() - t0
    return {"value": round(done / spent / 1e9, 6), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"rounds of {cores} x one layer's 7 projections at batch {m} over {cores} "
                      f"spawned processes ({spent:.1f} s)"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from i2_mpgemm_b200 import inputs
    m = args.batch
    sample, unit, work, what = oracle_sample(inputs, args.config, m)
    for _ in range(args.warmup):
        oracle_pass(sample)
    secs = [oracle_pass(sample)[0] for _ in range(args.steps)]
    total = sum(secs)
    value = rate(args.steps * work, total, unit)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": DATA,
        "config": workload_config(args.config, m, args.layers, args.gpus),
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": 1, "kind": "oracle",
                         "sample": f"each step: {what}, scalar C oracle, one thread"},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


DATA = ("synthetic (seeded ternary weights p=.25/.5/.25 x U(0.5,2) scale, N(0,1) activations)")


def workload_config(config: int, m: int, layers: int = 30, world: int = 1):
    """The `config` object of the JSON line, identical for both arms."""
    par = f"replicas x{world} (data parallel, no collective)"
    if config == 0:
        copies = kproj_copies()
        return {"workload": (f"k_proj GEMV 640x2560 at batch {m}, fused act-quant + I2_S matmul: "
                             f"{copies} distinct packed copies per step in one batched call"),
                "global_batch": m * world, "packed_bytes_per_step": copies * 640 * 2560 // 4,
                "l2": "inputs larger than L2: the copies total over 4x L2",
                "parallelism": par}
    if config == 1:
        return {"workload": ("one BitNet-b1.58-2B-4T layer's 7 projections at batch "
                             f"{m}, 1% outlier channels x20, fused act-quant + I2_S matmul, "
                             f"one call per step rotating over {LAYER_COPIES} layer copies"),
                "global_batch": m * world,
                "packed_bytes_per_step": sum(n * k // 4 for n, k in STACK_SHAPES),
                "l2": f"rotation over {LAYER_COPIES} distinct copies ({LAYER_COPIES} x 17.4 MB) "
                      "exceeds L2",
                "parallelism": par}
    if config == 3:
        return {"workload": (f"prefill GEMM at M={m}: gate/up 6912x2560 and down 2560x6912, "
                             "fused act-quant + tcgen05 int8 matmul, one batched call per step"),
                "global_batch": m * world,
                "int_ops_per_step": 2 * m * (2 * 6912 * 2560 + 2560 * 6912),
                "l2": "weights and activations L2-resident: tensor-bound by design",
                "parallelism": par}
    if config == 4:
        copies = 2 if m == 1 else 1
        return {"workload": (f"large BitNet-style layer (hidden 8192, ffn 28672), {copies} "
                             f"copies of its 7 projections at batch {m}, fused act-quant + I2_S "
                             "matmul in one batched call per step"),
                "global_batch": m * world,
                "packed_bytes_per_step": copies * LARGE_LAYER_BYTES,
                "l2": "inputs larger than L2 (214 MB per copy)",
                "parallelism": par}
    return {
        "workload": (f"BitNet-b1.58-2B-4T projection stack, {layers} layers x 7 "
                     "(q/o 2560x2560, k/v 640x2560, gate/up 6912x2560, down 2560x6912), "
                     f"decode batch {m}, fused act-quant + I2_S matmul per projection"),
        "global_batch": m * world,
        "packed_bytes_per_step": layers * sum(n * k // 4 for n, k in STACK_SHAPES),
        "l2": "inputs larger than L2: each step streams all packed weights (521 MB for 30 "
              "layers) from HBM",
        "parallelism": par,
    }


LAYER_COPIES = 16
# K of the problems of each of the four dependent calls of one layer
STAGE_KS = [[2560] * 3, [2560], [2560] * 2, [6912]]
LARGE_LAYER_BYTES = (2 * 8192 * 8192 + 2 * 1024 * 8192 + 3 * 28672 * 8192) // 4


def kproj_copies() -> int:
    return int(4 * L2_BYTES / (640 * 2560 // 4)) + 1


# ----------------------------------------------------------------- extras

def int8_gemm_tops(torch):
    """Dense int8 GEMM throughput of the library GEMM behind torch._int_mm
    (cuBLASLt) at 8192^3, best of 10 launches, or None where it is refused.
    A measurement of the tensor-core peak only; nothing on the path uses it."""
    n = 8192
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda")
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda")
        for bb in (b.t().contiguous().t(), b):
            try:
                torch._int_mm(a, bb)
                torch.cuda.synchronize()
                break
            except RuntimeError:
                bb = None
        if bb is None:
            return None
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, bb)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return 2.0 * n ** 3 / best / 1e9
    except Exception:  # an unsupported build or device: no measured peak
        return None


def int8_peak(torch, peaks):
    """(TOPS, source): the measured int8 GEMM, else bf16 burst x 2."""
    measured = int8_gemm_tops(torch)
    if measured:
        return measured, "measured: torch._int_mm 8192^3 best of 10"
    return (NOMINAL_INT8_OVER_BF16 * peaks["bf16_tflops"],
            f"{peaks['source']} bf16 burst x 2 (nominal int8/bf16 ratio)")


def gpu_ternary(torch, n: int, k: int, seed: int, scale=None):
    """Seeded ternary weights drawn on the device (same distribution as the
    host generator: -1/0/+1 with p = .25/.5/.25, times s ~ U(0.5, 2) or the
    given scale), for timing-only workloads whose host generation would take
    minutes."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    r = torch.randint(0, 4, (n, k), generator=g, device="cuda", dtype=torch.int32)
    s = 0.5 + 1.5 * torch.rand((), generator=g, device="cuda") if scale is None else scale
    return ((r == 3).float() - (r == 0).float()) * s


class Workload:
    """A config's timed work: `steps` is a list of steps, each a list of
    Problem run by one batched fused call; step i of a run uses
    steps[i % len(steps)].  All inputs sit in one Buffers."""

    def __init__(self, i2s, torch, steps, buf, unit, work_per_step, launches_per_step):
        self.i2s, self.torch = i2s, torch
        self.steps, self.buf, self.unit = steps, buf, unit
        self.work = work_per_step
        self.launches = launches_per_step
        self.plans = [stack_batch(i2s, probs) for probs in steps]
        self.ranges = []  # per step: (x lo, x hi, y lo, y hi) in the buffers
        for probs in steps:
            xs = [p.x.data_ptr() for p in probs]
            ys = [p.y.data_ptr() for p in probs]
            xb, yb = buf.x_dev.data_ptr(), buf.y_dev.data_ptr()
            xlo = (min(xs) - xb) // 4
            xhi = max((p.x.data_ptr() - xb) // 4 + p.x.numel() for p in probs)
            ylo = (min(ys) - yb) // 4
            yhi = max((p.y.data_ptr() - yb) // 4 + p.y.numel() for p in probs)
            self.ranges.append((xlo, xhi, ylo, yhi))

    def graphs(self):
        return [capture(self.torch, pl.run) for pl in self.plans]

    def h2d(self, i):
        lo, hi, _, _ = self.ranges[i % len(self.ranges)]
        self.buf.x_dev[lo:hi].copy_(self.buf.x_host[lo:hi], non_blocking=True)

    def d2h(self, i):
        _, _, lo, hi = self.ranges[i % len(self.ranges)]
        self.buf.y_host[lo:hi].copy_(self.buf.y_dev[lo:hi], non_blocking=True)

    def io_bytes(self):
        lo, hi, ylo, yhi = self.ranges[0]
        return 4 * (hi - lo), 4 * (yhi - ylo)


def problems_from_weights(i2s, torch, buf, specs, m):
    """Problems of (packed or fp32 weights, n, k, x host) specs in `buf`."""
    probs = []
    for w_or_packed, n, k, xh in specs:
        x, y, xhv = buf.take(m, k, n)
        xhv.copy_(xh.reshape(-1))
        if w_or_packed.dtype == torch.uint8:
            probs.append(Problem(i2s, torch, n, k, m, None, x, y, packed=w_or_packed))
        else:
            probs.append(Problem(i2s, torch, n, k, m, w_or_packed, x, y))
    return probs


def build_workload(i2s, torch, inputs, config: int, m: int, layers: int, rank: int):
    """The timed Workload of a config (each rank draws its own activations)."""
    off = 7919 * rank
    if config == 2:
        st = Stack(i2s, torch, inputs, layers, m, act_seed_offset=off)
        return Workload(i2s, torch, [st.probs], st.buf, "GB/s",
                        sum(p.packed_bytes for p in st.probs),
                        step_launches(m, [p.k for p in st.probs]))
    if config == 1:
        # LAYER_COPIES distinct copies of the layer (the same weights and
        # inputs), one call per step over one copy
        base = [(inputs.ternary_weights(p.n, p.k, inputs.seed_layer(idx))[0], p)
                for idx, p in enumerate(inputs.projections_2b())]
        xs = [inputs.activations(m, p.k, inputs.seed_layer(idx) + off, outliers=True)
              for idx, p in enumerate(inputs.projections_2b())]
        buf = Buffers(torch, LAYER_COPIES * sum(m * p.k for _, p in base),
                      LAYER_COPIES * sum(m * p.n for _, p in base))
        packs = [i2s.bitnet_i2s_pack(w.cuda()) for w, _ in base]
        steps = []
        for c in range(LAYER_COPIES):
            specs = [(pk if c == 0 else pk.clone(), p.n, p.k, x)
                     for pk, (_, p), x in zip(packs, base, xs)]
            steps.append(problems_from_weights(i2s, torch, buf, specs, m))
        buf.x_dev.copy_(buf.x_host)
        return Workload(i2s, torch, steps, buf, "GB/s", sum(n * k // 4 for n, k in STACK_SHAPES),
                        step_launches(m, [p.k for _, p in base]))
    if config == 0:
        copies = kproj_copies()
        w, _, _ = inputs.ternary_weights(640, 2560, inputs.seed_single())
        x = inputs.activations(m, 2560, inputs.seed_single() + off)
        pk = i2s.bitnet_i2s_pack(w.cuda())
        buf = Buffers(torch, copies * m * 2560, copies * m * 640)
        specs = [(pk if c == 0 else pk.clone(), 640, 2560, x) for c in range(copies)]
        probs = problems_from_weights(i2s, torch, buf, specs, m)
        buf.x_dev.copy_(buf.x_host)
        return Workload(i2s, torch, [probs], buf, "GB/s", copies * 640 * 2560 // 4,
                        step_launches(m, [2560] * copies))
    if config == 3:
        shapes = [(6912, 2560), (6912, 2560), (2560, 6912)]
        buf = Buffers(torch, sum(m * k for _, k in shapes), sum(m * n for n, _ in shapes))
        specs = []
        for idx, (n, k) in enumerate(shapes):
            seed = inputs.seed_prefill(idx)
            specs.append((inputs.ternary_weights(n, k, seed)[0], n, k,
                          inputs.activations(m, k, seed + off)))
        probs = problems_from_weights(i2s, torch, buf, specs, m)
        buf.x_dev.copy_(buf.x_host)
        return Workload(i2s, torch, [probs], buf, "TOPS",
                        sum(2.0 * m * n * k for n, k in shapes), step_launches(m, [2560, 2560, 6912]))
    # config 4: device-drawn weights (host generation of 1.7 G weights would take minutes)
    large = inputs.projections_large()
    copies = 2 if m == 1 else 1
    buf = Buffers(torch, copies * sum(m * p.k for p in large), copies * sum(m * p.n for p in large))
    packs = []
    for idx, p in enumerate(large):
        w = gpu_ternary(torch, p.n, p.k, inputs.seed_large(idx))
        packs.append(i2s.bitnet_i2s_pack(w))
        del w
    torch.cuda.empty_cache()
    specs = []
    for c in range(copies):
        for idx, p in enumerate(large):
            specs.append((packs[idx] if c == 0 else packs[idx].clone(), p.n, p.k,
                          inputs.activations(m, p.k, inputs.seed_large(idx) + off)))
    probs = problems_from_weights(i2s, torch, buf, specs, m)
    buf.x_dev.copy_(buf.x_host)
    return Workload(i2s, torch, [probs], buf, "GB/s", copies * LARGE_LAYER_BYTES,
                    step_launches(m, [p.k for p in large] * copies))


def staged_problems(i2s, torch, inputs, layers: int, m: int):
    """A dependency-staged decode step over the stack's shapes: per layer
    four stages -- q+k+v on the layer input, o on q's output, gate+up on o's
    output, down on gate's output, whose output is the next layer's input.
    Weights are drawn on the device with a per-tensor scale of 1/sqrt(K/2),
    so that the values passed from stage to stage keep their size over 120
    stages instead of overflowing; the matmul is the same.  Returns
    (problems as (packed, N, K, X, Y, None) in order, their stage numbers,
    packed bytes, tensors to keep alive); a problem's X is the very tensor
    an earlier problem writes as Y, or the external layer-0 input."""
    P = {p.name: p for p in inputs.projections_2b()}
    keep, probs, stages, nbytes = [], [], [], 0
    h = torch.randn((m, P["q"].k), generator=torch.Generator(device="cuda").manual_seed(5),
                    device="cuda")
    keep.append(h)
    for layer in range(layers):
        def add(name, idx, x, stage):
            p = P[name]
            w = gpu_ternary(torch, p.n, p.k, inputs.seed_stack(layer, idx),
                            scale=float((p.k / 2) ** -0.5))
            pk = i2s.bitnet_i2s_pack(w)
            y = torch.empty((m, p.n), device="cuda")
            keep.extend([pk, y])
            probs.append((pk, p.n, p.k, x, y, None))
            stages.append(stage)
            return y
        st = 4 * layer
        yq = add("q", 0, h, st)
        add("k", 1, h, st)
        add("v", 2, h, st)
        yo = add("o", 3, yq, st + 1)
        yg = add("gate", 4, yo, st + 2)
        add("up", 5, yo, st + 2)
        h = add("down", 6, yg, st + 3)
        nbytes += sum(n * k // 4 for n, k in STACK_SHAPES)
    torch.cuda.empty_cache()
    return probs, stages, nbytes, keep


def staged_stack(i2s, torch, inputs, layers: int, m: int, staged=None):
    """The staged step as 4 x layers batched fused calls in order, each stage
    reading what the one before it wrote.  Returns (list of BatchedQuantGemv
    in order, packed bytes per step, tensors to keep alive)."""
    probs, stages, nbytes, keep = staged or staged_problems(i2s, torch, inputs, layers, m)
    calls = []
    for st in range(stages[-1] + 1):
        calls.append(i2s.BatchedQuantGemv([p for p, s in zip(probs, stages) if s == st], m))
    return calls, nbytes, keep


def staged_chain(i2s, torch, inputs, layers: int, m: int, staged=None):
    """The staged step as one bitnet_i2s_quant_gemv_chain call.  Returns
    (QuantGemvChain, packed bytes per step, tensors to keep alive)."""
    probs, stages, nbytes, keep = staged or staged_problems(i2s, torch, inputs, layers, m)
    return i2s.QuantGemvChain(probs, stages, m), nbytes, keep


def staged_chain_measurement(i2s, torch, inputs, layers, m, steps, peaks):
    """The dependency-staged step as one chain call: its time, and whether
    its outputs equal, bit for bit, those of the 4 x layers separate calls
    on the same weights and input."""
    staged = staged_problems(i2s, torch, inputs, layers, m)
    calls, sbytes, keep = staged_stack(i2s, torch, inputs, layers, m, staged)
    chain, _, _ = staged_chain(i2s, torch, inputs, layers, m, staged)
    ys = [p[4] for p in staged[0]]
    for c in calls:
        c.run()
    want = [y.clone() for y in ys]
    for y in ys:
        y.fill_(float("nan"))
    chain.run()
    torch.cuda.synchronize()
    same = all(torch.equal(a, b) for a, b in zip(ys, want))
    del want, calls
    g = capture(torch, chain.run)
    ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
    n = len(staged[0])
    res = {"problems": n, "stages": staged[1][-1] + 1, "ms_per_step": round(ms, 4),
           "packed_GBps": round(sbytes / ms / 1e6, 1),
           "frac_of_hbm_measured": round(sbytes / ms / 1e6 / peaks["hbm_gbs"], 4),
           "tokens_per_s": round(m * 1000.0 / ms, 1),
           "us_per_stage": round(1000.0 * ms / (staged[1][-1] + 1), 2),
           "launches_per_step": 1 + -(-n // 128),
           "matches_staged_calls": same}
    del g, chain, keep, staged
    return res


def extra_measurements(i2s, torch, inputs, args, work, g_head, peaks):
    out = {}
    steps = args.steps
    int8_tops, int8_src = int8_peak(torch, peaks)
    out["int8_peak_TOPS"] = round(int8_tops, 1)
    out["int8_peak_source"] = int8_src
    # sustained: the headline step replayed for about a second, clocks sampled
    ms_one = time_replays(torch, g_head, 20, 3, collective=False)
    n_sus = max(200, int(1000.0 / max(ms_one, 1e-3)))
    with ClockSampler(gpu_uuid(torch, torch.cuda.current_device())) as clk:
        ms = time_replays(torch, g_head, n_sus, 3, collective=False)
    samp = clk.samples()
    sus = {"steps": n_sus, "seconds": round(n_sus * ms / 1000, 3), "ms_per_step": round(ms, 4),
           "packed_GBps": round(work.work / ms / 1e6, 1),
           "frac_of_hbm_measured": round(work.work / ms / 1e6 / peaks["hbm_gbs"], 4)}
    if samp:
        mhz = [s[0] for s in samp]
        med = statistics.median(mhz)
        bins = {}
        for s in mhz:
            key = f"{int(s // 100) * 100}-{int(s // 100) * 100 + 99}"
            bins[key] = bins.get(key, 0) + 1
        sus.update({"clock_samples": len(samp), "sm_mhz_median": med,
                    "sm_mhz_bins": dict(sorted(bins.items())),
                    "power_w_median": statistics.median(s[2] for s in samp),
                    "reasons": sorted(set().union(*[s[3] for s in samp])),
                    "ms_x_median_mhz": round(ms * med, 2)})
    out["sustained"] = sus
    probs1 = work.steps[0]
    m1 = probs1[0].m
    # the stack as 210 separate fused calls (420 launches per step)
    g = capture(torch, lambda: stack_step(i2s, probs1))
    ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
    nbytes = sum(p.packed_bytes for p in probs1)
    out["stack_batch1_per_call"] = {"ms_per_step": round(ms, 4),
                                    "packed_GBps": round(nbytes / ms / 1e6, 1),
                                    "launches_per_step": 2 * len(probs1)}
    del g
    # dependency-staged decode: 120 ordered calls per step
    for m in (1, 16):
        calls, sbytes, keep = staged_stack(i2s, torch, inputs, args.layers, m)
        g = capture(torch, lambda: [c.run() for c in calls])
        ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
        out[f"stack_staged_batch{m}"] = {
            "calls_per_step": len(calls), "ms_per_step": round(ms, 4),
            "packed_GBps": round(sbytes / ms / 1e6, 1),
            "frac_of_hbm_measured": round(sbytes / ms / 1e6 / peaks["hbm_gbs"], 4),
            "tokens_per_s": round(m * 1000.0 / ms, 1),
            "launches_per_step": args.layers * sum(step_launches(m, ks) for ks in STAGE_KS)}
        del g, calls, keep
        torch.cuda.empty_cache()
    # the same dependency-staged step as one chain call (one or two tokens)
    for m in (1, 2):
        out[f"stack_staged_chain_batch{m}"] = staged_chain_measurement(
            i2s, torch, inputs, args.layers, m, steps, peaks)
        torch.cuda.empty_cache()
    # the stack at batch 2, 4 and 16 (one batched call per step)
    for m in (2, 4, 16):
        probs = build_stack(i2s, torch, inputs, args.layers, m, 0)
        plan = stack_batch(i2s, probs)
        g = capture(torch, plan.run)
        ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
        nbytes = sum(p.packed_bytes for p in probs)
        out[f"stack_batch{m}"] = {"ms_per_step": round(ms, 4), "packed_GBps": round(
            nbytes / ms / 1e6, 1), "frac_of_hbm_measured": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4),
            "tokens_per_s": round(m * 1000.0 / ms, 1)}
        del g, plan, probs
        torch.cuda.empty_cache()
    # prefill GEMM: gate/up 6912x2560 and down 2560x6912 at M = 512 and 2048
    pre = {}
    for m in (512, 2048):
        for idx, (name, n, k) in enumerate([("gate", 6912, 2560), ("up", 6912, 2560),
                                            ("down", 2560, 6912)]):
            seed = inputs.seed_prefill(idx)
            w, _, _ = inputs.ternary_weights(n, k, seed)
            x = inputs.activations(m, k, seed)
            packed = i2s.bitnet_i2s_pack(w.cuda())
            xq, xs = i2s.bitnet_act_quant_i8(x.cuda())
            y = torch.empty((m, n), device="cuda")
            g = capture(torch, lambda: i2s.bitnet_i2s_gemm(packed, n, k, xq, xs, y=y))
            ms = time_replays(torch, g, 20, 3, collective=False)
            tops = 2.0 * m * n * k / ms / 1e9
            pre[f"{name}_M{m}"] = {"us": round(ms * 1000, 2), "TOPS": round(tops, 1),
                                   "frac_of_int8_peak": round(tops / int8_tops, 4),
                                   "frac_of_int8_spec_4500": round(tops / 4500.0, 4)}
            del g
    out["prefill_gemm"] = pre
    # single k_proj GEMV (640 x 2560, batch 1): one fused call, L2-resident
    w, _, _ = inputs.ternary_weights(640, 2560, inputs.seed_single())
    x = inputs.activations(1, 2560, inputs.seed_single())
    pr = Problem(i2s, torch, 640, 2560, 1, w, x.cuda(), torch.empty((1, 640), device="cuda"))
    g = capture(torch, lambda: i2s.bitnet_i2s_quant_gemv(pr.packed, 640, 2560, pr.x, y=pr.y,
                                                         workspace=pr.ws))
    ms = time_replays(torch, g, 200, 10, collective=False)
    g100 = capture(torch, lambda: [i2s.bitnet_i2s_quant_gemv(pr.packed, 640, 2560, pr.x, y=pr.y,
                                                             workspace=pr.ws) for _ in range(100)])
    ms100 = time_replays(torch, g100, 5, 2, collective=False) / 100
    out["k_proj_single"] = {"us_per_call": round(ms100 * 1000, 2),
                            "us_per_graph_replay_of_one_call": round(ms * 1000, 2),
                            "note": "one fused call (two launches) on L2-resident weights "
                                    "(0.41 MB); us_per_call from a graph of 100 calls in a row"}
    del g, g100
    # the block-64 IQ2_BN_R4 decode matmul at one token: four copies of a
    # 28672 x 8192 weight (235 MB, over L2), one call each per step
    n4, k4, copies = 28672, 8192, 4
    w = gpu_ternary(torch, n4, k4, 40000)
    r4s = [i2s.bitnet_iq2bn_pack(w, r4=True)]
    del w
    r4s += [r4s[0].clone() for _ in range(copies - 1)]
    xq, xs = i2s.bitnet_act_quant_i8(inputs.activations(1, k4, 40000).cuda())
    ys = [torch.empty((1, n4), device="cuda") for _ in range(copies)]
    g = capture(torch, lambda: [i2s.bitnet_iq2bn_r4_gemv(r, n4, k4, xq, xs, y=y)
                                for r, y in zip(r4s, ys)])
    ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
    nbytes = copies * n4 * k4 // 4
    out["iq2bn_r4_gemv_M1"] = {"shape": f"{copies} x {n4}x{k4}", "ms_per_step": round(ms, 4),
                               "packed_GBps": round(nbytes / ms / 1e6, 1),
                               "frac_of_hbm_measured": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4)}
    del g, r4s, ys
    torch.cuda.empty_cache()
    # the other GEMV configs, one line each: 0 (k_proj streamed), 1 (one
    # layer with outliers over 16 copies), 4 (large layer at M = 1 and 64)
    for cfg, m in ((0, 1), (1, 1), (4, 1), (4, 64)):
        wl = build_workload(i2s, torch, inputs, cfg, m, args.layers, 0)
        gs = wl.graphs()
        ms = time_replays(torch, gs, max(16, steps // 2), 3, collective=False)
        key = {0: "k_proj_streamed", 1: "config1_layer_outliers", 4: f"large_layer_M{m}"}[cfg]
        ent = {"ms_per_step": round(ms, 4), "packed_GBps": round(_packed(wl) / ms / 1e6, 1),
               "frac_of_hbm_measured": round(_packed(wl) / ms / 1e6 / peaks["hbm_gbs"], 4),
               "tokens_per_s": round(m * 1000.0 / ms, 1)}
        if cfg == 4:
            ops = sum(2.0 * m * p.n * p.k for p in wl.steps[0])
            ent["TOPS"] = round(ops / ms / 1e9, 1)
            ent["frac_of_int8_peak"] = round(ops / ms / 1e9 / int8_tops, 4)
        out[key] = ent
        del gs, wl
        torch.cuda.empty_cache()
    return out


def _packed(wl) -> int:
    return sum(p.packed_bytes for p in wl.steps[0])


# ------------------------------------------------------------------- main

def run_native(args):
    import numpy as np
    import torch

    from i2_mpgemm_b200 import i2s, inputs

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dist_init("nccl" if world > 1 else "gloo")
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()
    m = args.batch
    cfg_id = args.config
    if cfg_id != 3 and not 1 <= m <= 64:
        raise SystemExit("--batch must be in 1..64 for the decode configs")

    # Each rank: a replica of the weights, its own activations.
    work = build_workload(i2s, torch, inputs, cfg_id, m, args.layers, rank)
    # One CUDA graph per step of the rotation; step i replays graph i mod the
    # rotation (W warm-up steps, then the K timed ones).
    graphs = work.graphs()
    with ClockSampler(gpu_uuid(torch, local_rank)) as clk:
        ms = time_replays(torch, graphs, args.steps, args.warmup)
    ms = max_over_ranks(ms, dev)
    clocks = clk.summary()
    scale = 1e6 if work.unit == "GB/s" else 1e9
    value = world * work.work / ms / scale

    # End to end through the public API: every step copies that step's
    # inputs from pinned host memory to the device (one copy), runs the step
    # and copies its outputs back (one copy).
    h2d, d2h = work.io_bytes()
    ms_e2e = time_replays(torch, graphs, args.steps, args.warmup, before=work.h2d, after=work.d2h)
    ms_e2e = max_over_ranks(ms_e2e, dev)
    value_e2e = world * work.work / ms_e2e / scale

    # Roofline of the dominant kernel (the matmul), per launch.
    dp4a = all((m <= 2 and p.k <= 8192) or (m == 1 and p.k <= 30720) for p in work.steps[0])
    if work.unit == "GB/s":
        k_ms, k_launches, k_bytes = matmul_kernel_time(i2s, torch, work.steps)
        achieved = k_bytes / (k_ms / 1000.0) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": measured_traffic() if (dp4a and cfg_id == 2 and m == 1) else None,
                    "peak_source": peaks["source"],
                    "kernel": ("i2s_gemv_dp4a_kernel (persistent launches of up to 160 problems)"
                               if dp4a else
                               ("i2s_mma_kernel (persistent launches of up to 96 problems)"
                                if m <= 32 else
                                "i2s_prefill_kernel, 64-token tiles (persistent launches of up "
                                "to 96 problems)")),
                    "launches_per_step": k_launches,
                    "bytes_per_launch": int(k_bytes // k_launches),
                    "launch_us_mean": round(1000 * k_ms / k_launches, 3)}
    else:
        int8_tops, int8_src = int8_peak(torch, peaks)
        k_ms, k_launches, _ = matmul_kernel_time(i2s, torch, work.steps)
        achieved = work.work / (k_ms / 1000.0) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(int8_tops, 1),
                    "unit": "TOPS", "frac": round(achieved / int8_tops, 4), "traffic": None,
                    "peak_source": int8_src,
                    "kernel": ((f"i2s_prefill_kernel, {prefill_tile(m)}-token tiles "
                                "(persistent tcgen05 kind::i8, both operands in shared memory)")
                               if m > 32 else "i2s_mma_kernel (persistent tcgen05 kind::i8)"),
                    "launches_per_step": k_launches,
                    "ops_per_launch": int(work.work // k_launches),
                    "launch_us_mean": round(1000 * k_ms / k_launches, 3)}

    # Secondary measurements: one process only (with more ranks the others
    # would wait at the final barrier longer than the process-group timeout),
    # and no collective inside.
    extra = {}
    if rank == 0 and world == 1 and not args.no_extra and cfg_id == 2 and m == 1:
        extra = extra_measurements(i2s, torch, inputs, args, work, graphs[0], peaks)
    if work.unit == "GB/s":
        extra["step_frac_of_hbm_peak"] = round(value / world / peaks["hbm_gbs"], 4)
        extra["step_frac_of_hbm_spec_8tbs"] = round(value / world / 8000.0, 4)
        extra["kernel_frac_of_hbm_spec_8tbs"] = round(achieved / 8000.0, 4)
    extra["tokens_per_s"] = round(world * m * 1000.0 / ms, 1)
    extra["tokens_per_s_note"] = ("independent problems in one call per step; "
                                  "extra.stack_staged_* gives the dependency-staged step")

    cpu = None
    if rank == 0 and world == 1:
        # the outputs of the timed step for the problems the oracle sample
        # runs (the first problems of step 0), for the parity check
        n_sample = {0: 1, 1: 7, 2: 7, 3: 3, 4: 7}[cfg_id]
        torch.cuda.synchronize()
        work.plans[0].run()
        torch.cuda.synchronize()
        probs = work.steps[0]
        w_large = None
        if cfg_id == 3:
            gpu_out = [p.y[:min(m, 4)].cpu().numpy() for p in probs[:n_sample]]
        elif cfg_id == 4:
            # the down projection of copy 0, on the weights the timed arm drew
            pd = inputs.projections_large()[6]
            gpu_out = [probs[6].y[:1].cpu().numpy()]
            w_large = gpu_ternary(torch, pd.n, pd.k, inputs.seed_large(6)).cpu()
            torch.cuda.empty_cache()
        else:
            gpu_out = [p.y.cpu().numpy() for p in probs[:n_sample]]
        cpu = cpu_baseline(inputs, cfg_id, m, args.cpu_seconds, gpu_out, w_large)
        del w_large
        if not args.no_extra and cfg_id == 2:
            extra["cpu_baseline_all_cores"] = cpu_baseline_all_cores(m, args.cpu_seconds / 2)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": work.unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": DATA,
        "config": workload_config(cfg_id, m, args.layers, world),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "parity_ok": None if cpu is None or "parity" not in cpu else cpu["parity"]["parity_ok"],
        "e2e": {"value": round(value_e2e, 1), "unit": work.unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4)},
        "gpu_launches": work.launches * args.steps,
        "clocks": clocks,
        "extra": extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs
    barrier()
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_prefill_only(args):
    """gate 6912x2560 x 2048 tokens on pre-quantized activations: one warm
    call, `warmup` then `steps` graph replays."""
    import torch

    from i2_mpgemm_b200 import i2s, inputs
    n, k, m = 6912, 2560, 2048
    seed = inputs.seed_prefill(0)
    w, _, _ = inputs.ternary_weights(n, k, seed)
    packed = i2s.bitnet_i2s_pack(w.cuda())
    xq, xs = i2s.bitnet_act_quant_i8(inputs.activations(m, k, seed).cuda())
    y = torch.empty((m, n), device="cuda")
    g = capture(torch, lambda: i2s.bitnet_i2s_gemm(packed, n, k, xq, xs, y=y))
    ms = time_replays(torch, g, max(1, args.steps), max(1, args.warmup))
    print(json.dumps({"workload": "prefill GEMM gate 6912x2560, M=2048", "us": round(ms * 1000, 2),
                      "TOPS": round(2.0 * m * n * k / ms / 1e9, 1)}))
    return 0


def run_chain_only(args):
    """The dependency-staged step (4 x layers stages) as one chain call:
    `warmup` then `steps` graph replays, outputs checked against the same
    stages run as separate batched calls."""
    import torch

    from i2_mpgemm_b200 import i2s, inputs
    m = args.batch if args.batch in (1, 2) else 1
    res = staged_chain_measurement(i2s, torch, inputs, args.layers, m, max(2, 2 * args.steps),
                                   load_peaks())
    res["workload"] = f"dependency-staged {args.layers}-layer step, one chain call, batch {m}"
    print(json.dumps(res))
    return 0 if res["matches_staged_calls"] else 1


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill_only:
        return run_prefill_only(args)
    if args.chain_only:
        return run_chain_only(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
