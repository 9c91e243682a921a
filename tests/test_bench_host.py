"""Host logic of the benchmark that needs no GPU: the clock sampler's parsing
of the monitoring tool's output (run against a stand-in script on PATH)."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_tool(tmp_path, lines, monkeypatch):
    """A stand-in for nvidia-smi that prints `lines` in turn, then repeats
    the last one every 20 ms."""
    script = tmp_path / "nvidia-smi"
    body = "".join(f'echo "{ln}"; sleep 0.02\n' for ln in lines)
    script.write_text("#!/bin/bash\n" + body +
                      f'while true; do echo "{lines[-1]}"; sleep 0.02; done\n')
    script.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}:{os.environ['PATH']}")


IDLE = "0, 600, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active"
LOAD = "0, 1890, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active"


def test_sampler_reports_the_loaded_samples_and_their_reasons(tmp_path, monkeypatch):
    _fake_tool(tmp_path, [IDLE, LOAD], monkeypatch)
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.15)
    out = c.stop()
    assert out["samples"] >= 2
    assert out["sm_mhz"] == 1890.0          # the pre-region idle sample is dropped
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_sampler_has_a_sample_even_for_a_very_short_region(tmp_path, monkeypatch):
    _fake_tool(tmp_path, [LOAD], monkeypatch)
    c = bench.ClockSampler(0)
    c.start()                               # returns once the first sample is in
    out = c.stop()
    assert out["samples"] >= 1 and out["sm_mhz"] == 1890.0


def test_sampler_without_the_tool_reports_nothing(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    c = bench.ClockSampler(0)
    c.start()
    assert c.stop() is None


def test_traffic_is_reported_only_for_the_kernel_source_it_was_taken_on(monkeypatch):
    from block_sparse_attention_sbsa_b200 import workloads as W
    w = W.CONFIGS["rbs128k"]
    rec = bench.NCU_ATTEND_TRAFFIC["rbs128k"]
    assert bench.attend_kernel_source(w) == rec["source"]
    same = bench.source_hash(rec["source"]) == rec["sha"]
    assert bench.measured_traffic(w) == (rec["bytes"] if same else None)
    monkeypatch.setattr(bench, "source_hash", lambda rel: "0" * 16)
    assert bench.measured_traffic(w) is None                   # any other source
    assert bench.measured_traffic(W.CONFIGS["gqa32k"]) is None  # never captured


def test_spread_reports_median_and_deciles():
    s = bench.spread([float(x) for x in range(1, 12)])
    assert s["median"] == 6.0 and s["p10"] == 2.0 and s["p90"] == 10.0 and s["mean"] == 6.0
