"""Host logic of bench.py without a GPU: every workload's oracle CPU
baseline (one thread and all host cores) returns a well-formed, positive
figure in the workload's unit; the reference arm prints one line whose
config is the device arm's and whose step time is measured; the launch note
names the kernels a step forks; traffic from a profile summary is used only
while the kernel's source is unchanged."""
import argparse
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("workload", sorted(bench.STEPS))
def test_cpu_baseline_every_workload(workload):
    r = bench.cpu_baseline(workload, budget_s=0.3)
    assert r is not None, f"no oracle timing for {workload}"
    step = bench.STEPS[workload]
    assert r["unit"] == step.unit and r["value"] > 0 and r["work"] > 0
    assert r["kind"] == "oracle" and r["cores"] == bench.host_threads() and r["sample"] and r["cpu"]
    one = r["one_core"]
    assert one["cores"] == 1 and one["value"] > 0 and one["unit"] == step.unit and one["sample"]


def test_run_phases_covers_every_unit_once():
    seen = []
    ph = bench.OraclePhase("units", 1000, 1.0, lambda lo, hi: seen.extend(range(lo, hi)))
    runs = bench.run_phases([ph], 0.25, 3)
    assert runs[0][0] == 250 and sorted(seen) == list(range(250))
    step_s, work = bench.extrapolate([ph], [(250, 2.0)])
    assert step_s == pytest.approx(8.0) and work == 1000.0


def test_reference_line(capsys):
    args = argparse.Namespace(workload="qat_backward", steps=2, warmup=1, ref_step_s=0.1)
    bench.run_reference(args, 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["config"] == bench.STEPS["qat_backward"].CONFIG
    assert 0 < line["ms_per_step"] < 60_000            # a measured sampled step, not an extrapolation
    assert line["cpu_baseline"]["cores"] == bench.host_threads()
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_launch_note_names_forked_kernels():
    note = bench.launch_note(object.__new__(bench.DsFp8Gemm))
    assert "quant_fp8_128x128 on a second stream" in note
    assert "quant_nvfp4_b on a second stream" in bench.launch_note(object.__new__(bench.Nvfp4Gemm))
    assert "second stream" not in bench.launch_note(object.__new__(bench.MoeGrouped))


def test_whole_step_forks_side_kernels_before_the_first_kernel(monkeypatch):
    """The side kernels must not wait for the kernels listed before them:
    the side stream is forked from the current stream before the step's
    first kernel, and joined back just before `join_before`."""
    log = []

    class FakeStream:
        def __init__(self, name):
            self.name = name

        def wait_stream(self, other):
            log.append(f"{self.name} waits {other.name}")

    main, side = FakeStream("main"), FakeStream("side")
    current = [main]

    class Ctx:
        def __init__(self, s):
            self.s = s

        def __enter__(self):
            self.prev = current[0]
            current[0] = self.s

        def __exit__(self, *a):
            current[0] = self.prev

    monkeypatch.setattr(bench.torch.cuda, "current_stream", lambda: current[0])
    monkeypatch.setattr(bench.torch.cuda, "stream", lambda s: Ctx(s))

    class Step(bench.Step):
        side = ("b",)
        join_before = "g"

        def kernels(self):
            run = lambda n: (lambda: log.append(f"{n} on {current[0].name}"))
            return [("a", run("a")), ("b", run("b")), ("g", run("g")), ("h", run("h"))]

    Step().whole_step(side)
    assert log == ["side waits main", "a on main", "b on side", "main waits side", "g on main", "h on main"]


def test_traffic_only_for_unchanged_source(tmp_path, monkeypatch):
    h = bench._source_hash("moe_dispatch_mxfp8")
    assert h
    (tmp_path / "profiles").mkdir()
    f = tmp_path / "profiles" / "moe_dispatch_mxfp8__moe_dispatch.md"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "_source_hash", lambda kernel: h)   # the real source's hash
    f.write_text(f"source_sha256_16: {h}\ndram_bytes_per_launch: 123456\n")
    assert bench._traffic("moe_dispatch_mxfp8", "moe_dispatch") == 123456.0
    f.write_text("source_sha256_16: 0000000000000000\ndram_bytes_per_launch: 123456\n")
    assert bench._traffic("moe_dispatch_mxfp8", "moe_dispatch") is None
