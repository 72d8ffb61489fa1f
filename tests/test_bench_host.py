"""Host-side logic of bench.py (no GPU): the clock-sample summary, the recorded-traffic
lookup that goes null when a kernel source changes, and the algorithmic byte counts."""
import hashlib
import json
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(tmp_path, lines, uuid="GPU-aaaa"):
    path = tmp_path / "clocks.csv"
    path.write_text("".join(line + "\n" for line in lines))
    cs = bench.ClockSampler(uuid)
    cs.proc = _DoneProc()
    cs.path = str(path)
    return cs


def test_clock_summary_median_max_and_reasons(tmp_path, monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    row = "{u}, {sm}, 1965, 700.0, 0x0, {hw}, Not Active, Not Active, {cap}"
    lines = [row.format(u="GPU-aaaa", sm=1965, hw="Not Active", cap="Not Active"),
             row.format(u="GPU-aaaa", sm=1900, hw="Not Active", cap="Active"),
             row.format(u="GPU-aaaa", sm=1950, hw="Not Active", cap="Not Active"),
             # another GPU of the machine: ignored
             row.format(u="GPU-bbbb", sm=300, hw="Active", cap="Not Active"),
             "garbage line"]
    out = _sampler_with(tmp_path, lines).stop()
    assert out["sm_mhz"] == 1950
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 3


def test_clock_summary_flags_hardware_slowdown(tmp_path, monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    lines = ["GPU-aaaa, 1200, 1965, 900.0, 0x8, Active, Not Active, Active, Not Active"]
    out = _sampler_with(tmp_path, lines).stop()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples(tmp_path, monkeypatch):
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    out = _sampler_with(tmp_path, ["GPU-bbbb, 1965, 1965, 1, 0x0, a, b, c, d"]).stop()
    assert out["sm_mhz"] is None and out["reasons"] == ["no samples"]


def _fake_root(tmp_path, sources, recorded_bytes, tamper=False):
    (tmp_path / "profiles").mkdir()
    hs = hashlib.sha256()
    for name, text in sources.items():
        (tmp_path / name).write_text(text)
        hs.update(text.encode())
    entry = {"sources": list(sources), "source_hash": hs.hexdigest()[:16],
             "dram_bytes_per_launch": recorded_bytes}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"prefill": entry}))
    if tamper:
        first = next(iter(sources))
        (tmp_path / first).write_text(sources[first] + "// edited\n")
    return str(tmp_path)


def test_recorded_traffic_matches_the_captured_sources(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, {"a.cu": "kernel a\n", "b.cuh": "helpers\n"}, 1000)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.recorded_traffic("prefill") == 1000
    assert bench.recorded_traffic("decode") is None
    # scaled by the token count from the capture's T
    assert bench.prefill_traffic(bench.PREFILL_TRAFFIC_T // 2) == 500


def test_recorded_traffic_goes_null_after_a_source_edit(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, {"a.cu": "kernel a\n", "b.cuh": "helpers\n"}, 1000, tamper=True)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.recorded_traffic("prefill") is None
    assert bench.prefill_traffic(131072) is None


def test_algorithmic_bytes():
    # q, k, v, o bf16 (4 x 256 B) + log alpha fp32 (512 B) + beta (4 B) per token and head
    assert bench.PREFILL_BYTES_PER_TOKEN_HEAD == 4 * 256 + 512 + 4
    assert bench.prefill_bytes(131072, 32) == 131072 * 32 * 1540 + 32 * 65536
    # the head-wise gate reads one fp32 per token and head instead of d_k of them
    assert bench.prefill_bytes_head_gate(1, 1) == 1032 + 65536
    # decode: state read + write, q, k, v, log alpha, beta, o
    assert bench.DECODE_ACTIVE_BYTES == 132612


@pytest.mark.parametrize("T", [4096, 131072])
def test_prefill_roofline_time_is_bytes_over_copy_bandwidth(T):
    # 91.6 flop/B is below the ridge of the measured peaks, so the bound is the bytes
    flops = 141013.0 * T * 32
    nbytes = bench.prefill_bytes(T, 32)
    assert flops / nbytes < 1629e12 / 6548.2e9
