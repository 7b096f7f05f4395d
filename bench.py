#!/usr/bin/env python
"""Benchmark of the I2_S ternary x int8 matmul on B200.

Default workload (the JSON line's `value`): one decode step of the full
BitNet-b1.58-2B-4T projection stack -- 30 layers x 7 projections (q/o
2560x2560, k/v 640x2560, gate/up 6912x2560, down 2560x6912) = 210 fused
activation-quant + ternary matmuls at batch 1, each with its own seeded
fp32 input.  The 521 MB of packed weights stay resident in HBM; the working
set is over 4x the 126 MB L2, so every step streams them from HBM.  One step
is one replay of a CUDA graph holding one call of the public C ABI,
bitnet_i2s_quant_gemv_batched, over the 210 problems (at batch 1 and 2 that
is two launches: the activation quantizer and one persistent matmul).
`value` is packed-weight GB/s over all ranks.

Other measurements land in `extra`: the same stack as 210 separate
bitnet_i2s_quant_gemv calls, the stack at batch 2, 4 and 16, the prefill
GEMM (gate/up/down at M = 512 and 2048) in TOPS, and the single k_proj GEMV
latency.

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
# (N, K) of the seven projections of one BitNet-b1.58-2B-4T block
STACK_SHAPES = [(2560, 2560), (640, 2560), (640, 2560), (2560, 2560), (6912, 2560), (6912, 2560),
                (2560, 6912)]
TRAFFIC_SUMMARY = os.path.join(ROOT, "profiles", "i2s_gemv_dp4a_stack_batch1.md")
DECODE_SOURCES = [os.path.join(ROOT, "i2_mpgemm_b200", "csrc", f)
                  for f in ("gemv_kernel.cuh", "ptx.cuh")]


# ------------------------------------------------------------------ setup

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--batch", type=int, default=1, help="decode tokens per step (1..64)")
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary measurements")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the gate 6912x2560 prefill GEMM at M=2048 (a small case "
                         "for profiling the tensor-core kernel) and print its own line")
    return ap.parse_args(argv)


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

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def gpu_uuid(torch, device_index: int) -> str | None:
    try:
        u = str(torch.cuda.get_device_properties(device_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# ------------------------------------------------------------- workloads

class Problem:
    """One projection: resident packed weights plus views of the step buffers."""

    def __init__(self, i2s, torch, n, k, m, w, x, y):
        self.n, self.k, self.m = n, k, m
        self.packed = i2s.bitnet_i2s_pack(w.cuda())
        self.packed_bytes = n * k // 4
        self.x, self.y = x, y
        self.ws = torch.empty(i2s.bitnet_i2s_quant_gemv_workspace_bytes(m, k), dtype=torch.uint8,
                              device="cuda")


class Stack:
    """The projection stack with every input in one device buffer and every
    output in another (each problem's X and Y are views), so an end-to-end
    step moves its inputs and outputs with one copy each way."""

    def __init__(self, i2s, torch, inputs, layers: int, m: int, act_seed_offset: int):
        shapes = [(layer, idx, p) for layer in range(layers)
                  for idx, p in enumerate(inputs.projections_2b())]
        x_total = sum(m * p.k for _, _, p in shapes)
        y_total = sum(m * p.n for _, _, p in shapes)
        self.x_dev = torch.empty(x_total, dtype=torch.float32, device="cuda")
        self.y_dev = torch.empty(y_total, dtype=torch.float32, device="cuda")
        self.x_host = torch.empty(x_total, dtype=torch.float32).pin_memory()
        self.y_host = torch.empty(y_total, dtype=torch.float32).pin_memory()
        self.probs = []
        xo = yo = 0
        for layer, idx, p in shapes:
            seed = inputs.seed_stack(layer, idx)
            w, _, _ = inputs.ternary_weights(p.n, p.k, seed)
            xv = inputs.activations(m, p.k, seed + act_seed_offset)
            self.x_host[xo:xo + m * p.k].copy_(xv.reshape(-1))
            x = self.x_dev[xo:xo + m * p.k].view(m, p.k)
            y = self.y_dev[yo:yo + m * p.n].view(m, p.n)
            self.probs.append(Problem(i2s, torch, p.n, p.k, m, w, x, y))
            xo += m * p.k
            yo += m * p.n
            del w
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
    """Milliseconds per replay, CUDA events on the replay stream.  With
    `collective`, every rank must call it (barriers before and after);
    rank-0-only measurements pass collective=False."""
    for _ in range(warmup):
        if before:
            before()
        g.replay()
        if after:
            after()
    torch.cuda.synchronize()
    if collective:
        barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        if before:
            before()
        g.replay()
        if after:
            after()
    end.record()
    end.synchronize()
    torch.cuda.synchronize()
    if collective:
        barrier()
    return start.elapsed_time(end) / steps


def matmul_kernel_time(i2s, torch, probs, reps: int = 20):
    """Average device time of the matmul launch(es) of one step, CUDA events
    on the launching stream, with the activations quantized beforehand so the
    timed region holds only the matmul kernel.  Returns (ms per step,
    launches per step, algorithmic bytes per step)."""
    qs = [i2s.bitnet_act_quant_i8(p.x) for p in probs]
    m = probs[0].m
    plan = i2s.BatchedGemv([(p.packed, p.n, p.k, q, s, p.y, None)
                            for p, (q, s) in zip(probs, qs)], m)
    # The decode kernel takes up to DECODE_BATCH problems per launch (M <= 2,
    # K <= 8192, or M = 1 with K <= 30720), the tensor-core kernel up to
    # MMA_BATCH; the call also zeroes
    # the decode launches' work counters (one memset, inside the timed region).
    small = [p for p in probs if (m <= 2 and p.k <= 8192) or (m == 1 and p.k <= 30720)]
    launches = -(-len(small) // DECODE_BATCH) + -(-(len(probs) - len(small)) // MMA_BATCH)
    for _ in range(3):
        plan.run()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        plan.run()
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / reps
    nbytes = sum(p.packed_bytes + 4 + p.m * p.k + 4 * p.m + 4 * p.m * p.n for p in probs)
    return ms, launches, nbytes


# ------------------------------------------------------------ CPU oracle

def oracle_layer_sample(inputs, m: int):
    """One layer's seven projections packed by the oracle, with inputs."""
    import oracle
    sample = []
    for idx, p in enumerate(inputs.projections_2b()):
        seed = inputs.seed_stack(0, idx)
        w, _, _ = inputs.ternary_weights(p.n, p.k, seed)
        x = inputs.activations(m, p.k, seed)
        sample.append((oracle.pack(w.numpy()), p.n, p.k, x.numpy()))
    return sample


def oracle_layer_seconds(sample) -> float:
    import oracle
    t0 = time.perf_counter()
    for packed, n, k, x in sample:
        oracle.quant_gemm(packed, n, k, x)
    return time.perf_counter() - t0


def cpu_baseline(inputs, m: int, budget_s: float):
    sample = oracle_layer_sample(inputs, m)
    layer_bytes = sum(n * k // 4 for _, n, k, _ in sample)
    done, spent = 0, 0.0
    while spent < budget_s:
        spent += oracle_layer_seconds(sample)
        done += 1
    return {"value": round(done * layer_bytes / spent / 1e9, 6), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": f"{done} passes over one layer's 7 projections at batch {m} "
                      f"(scalar C oracle, one thread, {spent:.1f} s)"}


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
    sample = oracle_layer_sample(inputs, m)
    layer_bytes = sum(n * k // 4 for _, n, k, _ in sample)
    for _ in range(args.warmup):
        oracle_layer_seconds(sample)
    secs = [oracle_layer_seconds(sample) for _ in range(args.steps)]
    total = sum(secs)
    value = args.steps * layer_bytes / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": workload_config(args.layers, m),
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: one layer's 7 projections at batch {m} "
                                   "(1/30 of the stack), scalar C oracle, one thread"},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(layers: int, m: int):
    return {
        "workload": (f"BitNet-b1.58-2B-4T projection stack, {layers} layers x 7 "
                     "(q/o 2560x2560, k/v 640x2560, gate/up 6912x2560, down 2560x6912), "
                     f"decode batch {m}, fused act-quant + I2_S matmul per projection"),
        "global_batch": m,
        "packed_bytes_per_step": layers * sum(n * k // 4 for n, k in STACK_SHAPES),
        "l2": "inputs larger than L2: each step streams all packed weights (521 MB for 30 "
              "layers) from HBM",
        "parallelism": "replicas (data parallel, no collective)",
    }


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


def gpu_ternary(torch, n: int, k: int, seed: int):
    """Seeded ternary weights drawn on the device (same distribution as the
    host generator: -1/0/+1 with p = .25/.5/.25 times s ~ U(0.5, 2)), for the
    timing-only large layer whose host generation would take minutes."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    r = torch.randint(0, 4, (n, k), generator=g, device="cuda", dtype=torch.int32)
    s = 0.5 + 1.5 * torch.rand((), generator=g, device="cuda")
    return ((r == 3).float() - (r == 0).float()) * s


def extra_measurements(i2s, torch, inputs, steps: int, probs1, peaks):
    out = {}
    # int8 dense tensor peak: the library int8 GEMM measured here, else the
    # measured bf16 burst peak times the nominal int8/bf16 ratio of 2
    derived = 2.0 * peaks["bf16_tflops"]
    measured = int8_gemm_tops(torch)
    int8_tops = measured if measured else derived
    # the batch-1 stack as 210 separate fused calls (420 launches per step)
    g = capture(torch, lambda: stack_step(i2s, probs1))
    ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
    nbytes = sum(p.packed_bytes for p in probs1)
    out["stack_batch1_per_call"] = {"ms_per_step": round(ms, 4),
                                    "packed_GBps": round(nbytes / ms / 1e6, 1),
                                    "launches_per_step": 2 * len(probs1)}
    del g
    # the stack at batch 2, 4 and 16 (one batched call per step)
    for m in (2, 4, 16):
        probs = build_stack(i2s, torch, inputs, 30, m, 0)
        plan = stack_batch(i2s, probs)
        g = capture(torch, plan.run)
        ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
        nbytes = sum(p.packed_bytes for p in probs)
        out[f"stack_batch{m}"] = {"ms_per_step": round(ms, 4), "packed_GBps": round(
            nbytes / ms / 1e6, 1), "tokens_per_s": round(m * 1000.0 / ms, 1)}
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
    pre["int8_peak_TOPS"] = round(int8_tops, 1)
    pre["int8_peak_source"] = ("measured: torch._int_mm 8192^3 best of 10" if measured else
                               f"{peaks['source']} bf16 burst x 2 (nominal int8/bf16 ratio)")
    pre["int8_peak_derived_TOPS"] = round(derived, 1)
    out["prefill_gemm"] = pre
    # single k_proj GEMV (640 x 2560, batch 1): one launch vs graph steady state
    w, _, _ = inputs.ternary_weights(640, 2560, inputs.seed_single())
    x = inputs.activations(1, 2560, inputs.seed_single())
    pr = Problem(i2s, torch, 640, 2560, 1, w, x.cuda(), torch.empty((1, 640), device="cuda"))
    g = capture(torch, lambda: i2s.bitnet_i2s_quant_gemv(pr.packed, 640, 2560, pr.x, y=pr.y,
                                                         workspace=pr.ws))
    ms = time_replays(torch, g, 200, 10, collective=False)
    out["k_proj_single"] = {"us_per_call": round(ms * 1000, 2), "note": "L2-resident (0.41 MB)"}
    del g
    # k_proj streamed: distinct copies of the packed tensor totalling more
    # than 4x L2, one batched fused call per step
    copies = int(4 * 126e6 / (640 * 2560 // 4)) + 1
    xs_ = torch.empty((copies, 1, 2560), device="cuda").copy_(pr.x.view(1, 1, 2560).expand(copies, 1, 2560))
    ys_ = torch.empty((copies, 1, 640), device="cuda")
    pk = [pr.packed.clone() for _ in range(copies)]
    plan = i2s.BatchedQuantGemv([(pk[i], 640, 2560, xs_[i], ys_[i], None) for i in range(copies)], 1)
    g = capture(torch, plan.run)
    ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
    nbytes = copies * 640 * 2560 // 4
    out["k_proj_streamed"] = {"copies": copies, "ms_per_step": round(ms, 4),
                              "packed_GBps": round(nbytes / ms / 1e6, 1),
                              "frac_of_hbm_measured": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4)}
    del g, plan, pk, xs_, ys_
    torch.cuda.empty_cache()
    # large BitNet-style layer (hidden 8192, ffn 28672): two device copies of
    # its 7 projections (428 MB, more than 3x L2) at M = 1, and one at M = 64
    large = inputs.projections_large()
    packs = []
    for idx, p in enumerate(large):
        w = gpu_ternary(torch, p.n, p.k, inputs.seed_large(idx))
        packs.append(i2s.bitnet_i2s_pack(w))
        del w
    torch.cuda.empty_cache()
    layer_bytes = sum(p.n * p.k // 4 for p in large)
    for m, ncopy in ((1, 2), (64, 1)):
        probs, keep = [], []
        for c in range(ncopy):
            for idx, p in enumerate(large):
                pk = packs[idx] if c == 0 else packs[idx].clone()
                x = inputs.activations(m, p.k, inputs.seed_large(idx)).cuda()
                y = torch.empty((m, p.n), device="cuda")
                probs.append((pk, p.n, p.k, x, y, None))
        plan = i2s.BatchedQuantGemv(probs, m)
        g = capture(torch, plan.run)
        ms = time_replays(torch, g, max(5, steps // 2), 3, collective=False)
        nbytes = ncopy * layer_bytes
        ops = ncopy * sum(2.0 * m * p.n * p.k for p in large)
        out[f"large_layer_M{m}"] = {
            "layers": ncopy, "ms_per_step": round(ms, 4),
            "packed_GBps": round(nbytes / ms / 1e6, 1),
            "frac_of_hbm_measured": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4),
            "TOPS": round(ops / ms / 1e9, 1), "frac_of_int8_peak": round(ops / ms / 1e9 / int8_tops, 4),
            "tokens_per_s": round(m * 1000.0 / (ms / ncopy), 1)}
        del g, plan, probs
        torch.cuda.empty_cache()
    del packs
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------- main

def run_native(args):
    import torch

    from i2_mpgemm_b200 import i2s, inputs

    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dist_init("nccl" if world > 1 else "gloo")
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()
    m = args.batch
    if not 1 <= m <= 64:
        raise SystemExit("--batch must be in 1..64")

    # Each rank: a replica of the weights, its own activations.
    stack = Stack(i2s, torch, inputs, args.layers, m, act_seed_offset=7919 * rank)
    probs = stack.probs
    packed_bytes = sum(p.packed_bytes for p in probs)
    plan = stack_batch(i2s, probs)
    dp4a = m <= 2
    launches_per_step = step_launches(m, [p.k for p in probs])

    g = capture(torch, plan.run)
    with ClockSampler(gpu_uuid(torch, local_rank)) as clk:
        ms = time_replays(torch, g, args.steps, args.warmup)
    ms = max_over_ranks(ms, dev)
    clocks = clk.summary()
    value = world * packed_bytes / ms / 1e6  # GB/s over all ranks

    # End to end through the public API: every step copies all 210 inputs
    # from pinned host memory to the device (one copy), runs the step and
    # copies all outputs back (one copy).
    h2d = stack.x_dev.numel() * 4
    d2h = stack.y_dev.numel() * 4
    ms_e2e = time_replays(torch, g, args.steps, args.warmup, before=stack.h2d, after=stack.d2h)
    ms_e2e = max_over_ranks(ms_e2e, dev)
    value_e2e = world * packed_bytes / ms_e2e / 1e6

    # Roofline of the dominant kernel (the matmul), per launch.
    k_ms, k_launches, k_bytes = matmul_kernel_time(i2s, torch, probs)
    achieved = k_bytes / (k_ms / 1000.0) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": measured_traffic() if dp4a else None, "peak_source": peaks["source"],
                "kernel": ("i2s_gemv_dp4a_kernel (persistent launches of up to 160 problems)"
                           if dp4a else "i2s_mma_kernel (persistent launches of up to 96 problems)"),
                "launches_per_step": k_launches,
                "bytes_per_launch": int(k_bytes // k_launches),
                "launch_us_mean": round(1000 * k_ms / k_launches, 3)}

    # Secondary measurements: one process only (with more ranks the others
    # would wait at the final barrier longer than the process-group timeout),
    # and no collective inside.
    extra = {}
    if rank == 0 and world == 1 and not args.no_extra:
        extra = extra_measurements(i2s, torch, inputs, args.steps, probs, peaks)
    extra["step_frac_of_hbm_peak"] = round(value / world / peaks["hbm_gbs"], 4)
    extra["step_frac_of_hbm_spec_8tbs"] = round(value / world / 8000.0, 4)
    extra["kernel_frac_of_hbm_spec_8tbs"] = round(achieved / 8000.0, 4)
    extra["tokens_per_s"] = round(world * m * 1000.0 / ms, 1)

    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline(inputs, m, args.cpu_seconds)
        if not args.no_extra:
            extra["cpu_baseline_all_cores"] = cpu_baseline_all_cores(m, args.cpu_seconds / 2)

    cfg = workload_config(args.layers, m)
    cfg["packed_bytes_per_step"] = packed_bytes
    cfg["global_batch"] = m * world
    cfg["parallelism"] = f"replicas x{world} (data parallel, no collective)"
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded ternary weights p=.25/.5/.25 x U(0.5,2) scale, N(0,1) "
                "activations)",
        "config": cfg,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": round(value_e2e, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "extra": extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g
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


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill_only:
        return run_prefill_only(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
