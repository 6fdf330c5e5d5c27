"""Host logic of bench.py on the CPU: the reference arm's JSON line, the
algorithmic work per prefill and the traffic lookup that is only trusted
while the GEMM source is the one the ncu counters were taken on."""
import json
import os
import subprocess
import sys

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_complete_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "1",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True


def test_algorithmic_flops_of_the_headline_workload():
    """1.728e15 flop per 2.7B / 128K prefill (13.18 GFLOP per token): forward
    of every block, LM head, backward through the updated blocks, band-only
    attention (eq. (1) pair count)."""
    cfg = synth.get_config("2.7b")
    f = bench.algorithmic_flops(cfg, cfg.T)
    assert abs(f / 1.72779e15 - 1) < 1e-4, f
    assert abs(f / cfg.T / 1e9 - 13.18) < 0.01


def test_traffic_is_trusted_only_for_the_captured_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kc: "abc")
    assert bench.traffic_for("gemm", "2.7b") is None  # no file
    (prof / "traffic.json").write_text(json.dumps({"2.7b": {"gemm": {"source_hash": "abc",
                                                                     "dram_bytes_per_launch": 123}}}))
    assert bench.traffic_for("gemm", "2.7b") == 123
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kc: "changed")
    assert bench.traffic_for("gemm", "2.7b") is None


def test_latency_sweep_covers_prefixes_and_the_whole_sequence(monkeypatch):
    """latency_by_tokens prefills each shorter prefix once and the whole
    sequence once, from a fresh state each time, and reports ms per 1K
    tokens per length (fake context and events: no GPU)."""
    import types

    calls = []

    class Ctx:
        def reset(self):
            calls.append("reset")

        def prefill(self, tok, losses, sync=True):
            calls.append(("prefill", len(tok), len(losses), sync))

        def sync(self):
            calls.append("sync")

    class Event:
        t = 0.0

        def __init__(self, enable_timing=False):
            self.at = None

        def record(self, stream=None):
            Event.t += 5.0
            self.at = Event.t

        def elapsed_time(self, other):
            return other.at - self.at

    fake_torch = types.SimpleNamespace(cuda=types.SimpleNamespace(Event=Event))
    monkeypatch.setitem(sys.modules, "torch", fake_torch)
    out = bench.latency_by_tokens(Ctx(), list(range(40000)), list(range(40000)), 40000, None)
    assert list(out) == ["8192", "16384", "32768", "40000"]
    assert [c[1] for c in calls if isinstance(c, tuple)] == [8192, 16384, 32768, 40000]
    assert all(c[3] is False for c in calls if isinstance(c, tuple))
    assert calls.count("reset") == 4 and calls.count("sync") == 4
    assert abs(out["8192"] - 5.0 / 8.192) < 1e-12
