"""Host-side logic of bench.py that the reported numbers rest on (no GPU)."""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


class _FakeProc:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def _line(stamp, mhz, watts, cap):
    return f"{stamp}, {mhz}, 1965, {watts}, Not Active, Not Active, Not Active, {cap}"


def test_clock_samples_are_taken_inside_the_timed_region(bench, monkeypatch):
    """Idle samples before and after the timed region do not enter the median,
    and throttle reasons count only inside it."""
    s = bench.ClockSampler(0)
    base = bench.ClockSampler._stamp("2026/12/02 10:00:00.000")
    lines = [_line("2026/12/02 10:00:00.000", 1965, 240, "Not Active"),    # idle, before
             _line("2026/12/02 10:00:00.500", 1600, 990, "Active"),        # loaded
             _line("2026/12/02 10:00:00.700", 1580, 1000, "Active"),
             _line("2026/12/02 10:00:00.900", 1620, 980, "Active"),
             _line("2026/12/02 10:00:01.500", 1965, 250, "Not Active")]    # idle, after
    s.proc = _FakeProc("\n".join(lines))
    s.t0, s.t1 = base + 0.4, base + 1.0
    monkeypatch.setattr(bench.time, "sleep", lambda _: None)
    c = s.stop()
    assert c["samples"] == 3 and c["window"] == "timed region"
    assert c["sm_mhz"] == 1600 and c["power_w"] == 990
    assert c["reasons"] == ["sw_power_cap"] and c["sm_max_mhz"] == 1965


def test_short_region_falls_back_to_the_loaded_samples(bench, monkeypatch):
    s = bench.ClockSampler(0)
    base = bench.ClockSampler._stamp("2026/12/02 10:00:00.000")
    lines = [_line("2026/12/02 10:00:00.000", 1965, 240, "Not Active"),
             _line("2026/12/02 10:00:00.100", 1700, 900, "Active"),
             _line("2026/12/02 10:00:00.200", 1965, 245, "Not Active")]
    s.proc = _FakeProc("\n".join(lines))
    s.t0, s.t1 = base + 0.12, base + 0.15      # no sample falls inside
    monkeypatch.setattr(bench.time, "sleep", lambda _: None)
    c = s.stop()
    assert c["samples"] == 1 and c["sm_mhz"] == 1700 and c["window"].startswith("samples at")
    assert c["reasons"] == ["sw_power_cap"]


def test_without_nvidia_smi_the_clock_is_reported_missing(bench):
    s = bench.ClockSampler(0)
    s.proc = None
    assert s.stop()["reasons"] == ["nvidia-smi unavailable"]


def test_percentiles_are_nearest_rank(bench):
    xs = [5.0, 1.0, 4.0, 2.0, 3.0]
    assert bench.pct(xs, 50) == 3.0
    assert bench.pct(xs, 95) == 5.0
    assert bench.pct(xs, 0) == 1.0
    assert bench.pct([7.0], 95) == 7.0


def test_attention_denominator_is_the_burst_peak(bench):
    """The roofline divides by the larger (burst) GEMM figure; the sustained
    one is only reported beside it."""
    pk = {"hbm_gbs": 6549.4, "bf16_tflops": 1642.9, "bf16_tflops_sustained": 1392.3}
    assert bench.tensor_peak(pk) == (1642.9, "bf16 burst")
    assert bench.sustained_peak(pk) == 1392.3
    assert bench.tensor_peak({"bf16_tflops": 1590.0})[0] == 1590.0
    assert bench.sustained_peak({"bf16_tflops": 1590.0}) == 1590.0


def test_default_workload_is_the_largest_single_gpu_layer(bench):
    P, N, H, C, seed, cu = bench.WORKLOADS["long104k"]
    assert (P, N, H, C, seed, cu) == (8, 104_448, 56, 3, 3, None)
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert 'default="long104k"' in src


def test_both_oracle_legs_use_one_sample_definition(bench):
    """cpu_baseline and --impl reference call oracle_sample with the same
    defaults: 4096 rows per head of two heads, extrapolated x N/rows x H/heads."""
    import numpy as np
    from ulysses_sequence_attention_repack_b200 import inputs
    assert bench.ORACLE_ROWS_PER_HEAD == 4096 and bench.ORACLE_HEADS == 2
    S = inputs.qkv_seq(1024, 8, 2, 3, 0, "cpu")
    us, sample = bench.oracle_sample("tiny", inputs.host_bits(S))
    assert us > 0
    # N = 1024 <= 4096: every row of every head of rank 0, x 2 for rank 1's heads
    assert "1024 query rows x 4 heads" in sample and "x1.00 rows x 2.0 heads" in sample
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert "oracle_sample(args.config, S_bits)" in src and "oracle_sample(config, S_bits)" in src
    assert np.isfinite(us)


def test_algorithmic_flops(bench):
    # 4 N^2 H D for one sequence; varlen sums the segments; causal counts n + 1 keys per row
    assert bench.attn_flops(1024, 8, None) == 4 * 1024 ** 2 * 8 * 128
    assert bench.attn_flops(100, 2, [0, 60, 100]) == 4 * (60 ** 2 + 40 ** 2) * 2 * 128
    assert bench.attn_flops(4, 1, None, causal=True) == 4 * 128 * (4 * 5 // 2)


def test_traffic_record_is_void_once_the_source_changes(bench, tmp_path, monkeypatch):
    import json
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "ulysses_sequence_attention_repack_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k.cu").write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"k": {"w": {"source": "k.cu", "source_sha256_16": bench.source_hash("k.cu"), "dram_bytes_per_launch": 42}}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("k", "w") == 42
    (src / "k.cu").write_text("kernel v2")
    assert bench.recorded_traffic("k", "w") is None
    assert bench.recorded_traffic("k", "other") is None


def test_peer_pointer_table_keeps_the_tensor_offset():
    """PeerLayer maps its tensor's address on every rank from the symmetric
    allocation's base addresses plus the tensor's offset inside its own."""
    from ulysses_sequence_attention_repack_b200 import peer

    class Handle:
        buffer_ptrs = [0x7000_0000_0000, 0x7100_0000_0000, 0x7200_0000_0000]

    class Local:
        def data_ptr(self):
            return 0x7100_0000_0000 + 4096

    layer = peer.PeerLayer.__new__(peer.PeerLayer)
    layer.rank = 1
    layer.exchange = "symmetric"
    assert layer._peer_ptrs(Handle(), Local()) == [0x7000_0000_1000, 0x7100_0000_1000, 0x7200_0000_1000]
