"""Host-side logic of bench.py (CPU only): the algorithmic byte counts behind
the roofline, the whole-job aggregation, the clock-record parsing and the
hash-keyed ncu traffic lookup."""
import os

import bench
from linear_vision_backbone_b200 import inputs


def test_algorithmic_bytes_of_the_16k_step():
    wl = inputs.WORKLOADS["16k"]
    th = 16384 * 6
    ab = bench.alg_bytes(wl, 2)
    # K4: q, k, v, z (2 bytes x 64 each), g (4 x 64), out (2 x 64) per token-head: 896 bytes
    assert ab["output"] == th * 896
    # K2: k, v, g per token-head; K3 touches only the workspace
    assert ab["summary"] == th * (128 + 128 + 256)
    assert ab["scan"] == 0
    # K1: x once (384 x 2 bytes per token) and g written
    assert ab["gate"] == 16384 * 384 * 2 + th * 256
    # the fused gate: rank-16 rows instead of g in K1, read by K2 (which then writes g)
    fused = bench.alg_bytes(wl, 2, fused=True)
    assert fused["gate"] == 16384 * 384 * 2 + 16384 * 16 * 4
    assert fused["summary"] == ab["summary"] + 16384 * 16 * 4
    assert fused["output"] == ab["output"]
    # boundary states are workspace traffic, reported apart from the algorithmic bytes
    ws = bench.workspace_bytes(wl, 256)
    st = 6 * 256 * (64 * 64 + 64) * 4
    assert ws == {"gate": 0, "summary": st, "scan": 2 * st, "output": st}


def test_whole_step_algorithmic_bytes_of_every_workload():
    # gate + GLA at d = 64, 16-bit: 896 + 384 bytes per token-head (x is 384 x 2 / 6 heads)
    wl = inputs.WORKLOADS["16k"]
    assert bench.step_alg_bytes(wl) == wl.token_heads * (896 + 384)
    wl = inputs.WORKLOADS["640b8"]
    assert bench.step_alg_bytes(wl) == 8 * 1600 * 6 * (896 + 384)
    # GLA alone (gates drawn directly): d = 128 bf16 is 5 x 256 + 512 = 1792 bytes
    wl = inputs.WORKLOADS["sweep"].with_grid(64)
    assert bench.step_alg_bytes(wl) == 4096 * 4 * 1792
    # fp32 d = 16: 5 x 64 + 64 = 384 bytes
    wl = inputs.WORKLOADS["tiny"]
    assert bench.step_alg_bytes(wl) == 64 * 384


def test_host_cpu_record():
    h = bench.host_cpu()
    assert h["host_cores"] == os.cpu_count()
    assert "cpu_model" in h


def test_whole_job_value_counts_every_rank():
    # 98304 token-heads per rank per step, 10 steps in 1 ms on the slowest of 4 ranks
    assert bench.aggregate_value(98304, 10, 1.0, 4) == 4 * 98304 * 10 / 1e-3


class _FakeProc:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def test_clock_record_parsing():
    rows = [
        "0, 1965, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle
        "0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",      # power cap
        "0, 1900, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = bench.ClockSampler(0)
    s.proc = _FakeProc("\n".join(rows))
    c = s.stop()
    assert c["samples"] == 4 and c["samples_under_load"] == 3
    assert c["sm_mhz"] == 1900.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    s.proc = _FakeProc("")
    assert s.stop() is None


def test_traffic_lookup_is_keyed_by_the_kernel_source_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    f = tmp_path / "traffic.txt"
    f.write_text("# comment\n"
                 f"gla_out_tc:tc:16k {h} 123456 dram_read+write_bytes_per_launch\n"
                 "gla_sum_tc:tc:16k 000000000000 999 dram_read+write_bytes_per_launch\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.read_traffic("gla_out_tc:tc:16k", h) == (123456.0, "dram_read+write_bytes_per_launch")
    assert bench.read_traffic("gla_sum_tc:tc:16k", h) == (None, None)      # stale hash
    assert bench.read_traffic("gate_fwd_tc:tc:16k", h) == (None, None)     # absent


def test_kernel_source_hash_ignores_comments(tmp_path, monkeypatch):
    root = tmp_path
    csrc = root / "linear_vision_backbone_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cuh").write_text("int f() { return 1; }  // one\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    h1 = bench.kernel_source_hash()
    (csrc / "a.cuh").write_text("/* header */\nint f() {\n  return 1;   // another comment\n}\n")
    assert bench.kernel_source_hash() == h1
    (csrc / "a.cuh").write_text("int f() { return 2; }\n")
    assert bench.kernel_source_hash() != h1
    assert os.path.isdir(csrc)


def test_sswiglu_algorithmic_bytes():
    # u read once (2C channels), h written once (C channels), 16-bit; fp32 taps (9 C) and bias (C)
    assert bench.sswiglu_bytes(1, 16384, 1024) == 16384 * 3 * 1024 * 2 + 10 * 1024 * 4
    assert bench.sswiglu_bytes(2, 10, 8) == 2 * 10 * 24 * 2 + 80 * 4
