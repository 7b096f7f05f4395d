"""Host-side logic of bench.py, without a GPU: the launch count it reports,
the workload description it prints, the rule that ties the recorded
DRAM traffic to the kernel code it was captured on, and the warm-up of a
rotation of graphs."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


STACK_KS = [2560, 2560, 2560, 2560, 2560, 2560, 6912] * 30


def test_launches_per_step(bench):
    # batch 1 and 2: one quantizer launch, two decode launches (210 / 160)
    assert bench.step_launches(1, STACK_KS) == 3
    assert bench.step_launches(2, STACK_KS) == 3
    # batch 16: one quantizer launch, three tensor-core launches (210 / 96)
    assert bench.step_launches(16, STACK_KS) == 4
    # long K: one token stays on the decode kernel, two tokens do not
    assert bench.step_launches(1, [28672]) == 2
    assert bench.step_launches(2, [28672]) == 2
    assert bench.step_launches(1, [131072]) == 2
    assert bench.step_launches(1, [128] * 1001) == 2 + 7


def test_workload_config_counts_the_stack(bench):
    cfg = bench.workload_config(2, 1, 30)
    n_k = [(2560, 2560), (640, 2560), (640, 2560), (2560, 2560), (6912, 2560), (6912, 2560),
           (2560, 6912)]
    assert cfg["packed_bytes_per_step"] == 30 * sum(n * k // 4 for n, k in n_k) == 521011200


def test_code_digest_ignores_comments_only(bench, tmp_path):
    a = tmp_path / "a.cuh"
    a.write_text("int f(int x) {  // one\n  return x + 1;\n}\n/* block\n comment */\n")
    b = tmp_path / "b.cuh"
    b.write_text("// header\n\nint f(int x) {\n  return x + 1;   \n}\n")
    c = tmp_path / "c.cuh"
    c.write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.code_digest([a]) == bench.code_digest([b])
    assert bench.code_digest([a]) != bench.code_digest([c])


def test_recorded_traffic_is_dropped_when_the_code_changes(bench, tmp_path, monkeypatch):
    got = bench.measured_traffic()
    assert got is None or (isinstance(got, int) and got > 0)
    changed = []
    for path in bench.DECODE_SOURCES:
        dst = tmp_path / os.path.basename(path)
        dst.write_text(open(path).read() + "\nstatic const int kChanged = 1;\n")
        changed.append(str(dst))
    monkeypatch.setattr(bench, "DECODE_SOURCES", changed)
    assert bench.measured_traffic() is None


def test_every_config_has_a_workload_and_the_reference_arm_prints_the_same_config(bench):
    for c in range(5):
        m = bench.DEFAULT_BATCH[c]
        cfg = bench.workload_config(c, m, 30, 1)
        assert cfg["workload"] and cfg["global_batch"] == m
        assert cfg == bench.workload_config(c, m, 30, 1)
    args = bench.parse_args(["--config", "3"])
    assert args.batch == 2048
    assert bench.parse_args([]).config == 2 and bench.parse_args([]).batch == 1


def test_output_comparison_flags_a_wrong_or_nonzero_value(bench):
    import numpy as np
    want = [np.array([[1.0, 0.0, -2.0]], np.float32)]
    assert bench.compare_outputs([want[0].copy()], want)["parity_ok"]
    bad = want[0].copy()
    bad[0, 2] = -2.001
    assert not bench.compare_outputs([bad], want)["parity_ok"]
    bad = want[0].copy()
    bad[0, 1] = 1e-30
    assert not bench.compare_outputs([bad], want)["parity_ok"]


def test_reference_arm_line_on_a_small_sample(bench, capsys):
    # config 0 at batch 1: one k_proj problem per step through the oracle
    bench.run_reference(bench.parse_args(["--impl", "reference", "--config", "0", "--steps", "1",
                                          "--warmup", "0"]))
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["config"] == bench.workload_config(0, 1, 30, 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0


class _FakeCuda:
    """Records graph replays and event records in order (no GPU)."""

    def __init__(self, log):
        self.log = log

    def synchronize(self):
        pass

    def Event(self, enable_timing=False):
        log = self.log

        class _Ev:
            def record(self):
                log.append(("record",))

            def synchronize(self):
                pass

            def elapsed_time(self, other):
                return 1.0

        return _Ev()


class _FakeGraph:
    def __init__(self, log, idx):
        self.log, self.idx = log, idx

    def replay(self):
        self.log.append(("replay", self.idx))


def test_rotation_replays_every_graph_before_the_timed_region(bench):
    """A graph's first replay uploads it; with a rotation longer than the
    warm-up, every graph must still have been replayed once before the start
    event, and the timed region must replay exactly `steps` graphs."""
    import types
    log = []
    torch = types.SimpleNamespace(cuda=_FakeCuda(log))
    graphs = [_FakeGraph(log, i) for i in range(16)]
    ms = bench.time_replays(torch, graphs, steps=20, warmup=5, collective=False)
    start = log.index(("record",))
    before = {e[1] for e in log[:start] if e[0] == "replay"}
    assert before == set(range(16))
    timed = [e for e in log[start + 1:] if e[0] == "replay"]
    assert len(timed) == 20 and log[-1] == ("record",)
    assert ms == pytest.approx(1.0 / 20)
