"""Host-side pieces of bench.py that decide the reported numbers, checked without a GPU:
the algorithmic bytes behind the roofline, the parser of the clock record, and the
lookup of recorded DRAM traffic, which must only answer for the current kernel sources."""
import os

import bench
import workloads as W


# Hand counts per step at the first decode step's length (N0 + 1 tokens):
# summaries = units * nb * 4d bytes (a bf16 min row and max row per block), K and V of
# the K true top-K blocks = units * K * bs * d * 2 (bf16) * 2 (K and V).
HAND = {
    "llama8b_32k": 8 * 513 * 4 * 128 + 8 * 64 * 64 * 128 * 2 * 2,       # 18.88 MB
    "batched_128k": 128 * 1025 * 4 * 128 + 128 * 32 * 128 * 128 * 2 * 2,  # 335.6 MB
    "long_512k": 32 * 4097 * 4 * 128 + 32 * 64 * 128 * 128 * 2 * 2,     # 201.3 MB
}


def test_algorithmic_bytes_match_hand_counts():
    for name, want in HAND.items():
        w = W.workload(name)
        assert bench.algorithmic_bytes(w, w.N0 + 1)["total"] == want, name
    assert round(HAND["llama8b_32k"] / 1e6, 2) == 18.88
    assert round(HAND["batched_128k"] / 1e6, 1) == 335.6
    assert round(HAND["long_512k"] / 1e6, 1) == 201.3


def test_algorithmic_bytes_take_every_block_when_k_exceeds_them():
    w = W.workload("tiny")
    n = 2 * w.bs  # two blocks, K = 8 of them wanted
    got = bench.algorithmic_bytes(w, n)
    assert got["kv"] == w.units * 2 * w.bs * w.d * 4
    assert got["summaries"] == w.units * 2 * 4 * w.d


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def test_clock_record_parser():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.proc = _FakeProc()
    cs.lines = [
        "0, 1965, 1965, 650.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1305, 1965, 1000.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, 1000.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # skipped
        "short line",
    ]
    assert cs.stop() == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    cs.lines = ["0, 1200, 1965, 800.0, 0x8, Active, Not Active, Active, Not Active"]
    assert cs.stop()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_record_without_nvidia_smi():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.proc, cs.lines = None, []
    r = cs.stop()
    assert r["sm_mhz"] is None and r["samples"] == 0 and r["reasons"] == ["nvidia-smi unavailable"]


def test_recorded_traffic_only_for_the_current_kernel_sources(tmp_path, monkeypatch):
    os.makedirs(tmp_path / "profiles")
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# kernel workload sha bytes\n"
        "fused_step_kernel batched_128k cafe0000cafe0000 123456789\n"
        "fused_step_kernel long_512k 0123456789abcdef 5\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "cafe0000cafe0000")
    assert bench.recorded_traffic("fused_step_kernel", "batched_128k") == 123456789.0
    assert bench.recorded_traffic("fused_step_kernel", "long_512k") is None  # other sources
    assert bench.recorded_traffic("fused_step_kernel", "llama8b_32k") is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda: "0000000000000000")
    assert bench.recorded_traffic("fused_step_kernel", "batched_128k") is None


def test_kernel_source_sha_covers_every_kernel_source():
    csrc = os.path.join(bench.ROOT, "dynamic_sparse_attention_block_b200", "csrc")
    names = sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h")))
    assert "fused_step.cu" in names and "prr_schedule.h" in names
    sha = bench.kernel_source_sha()
    assert len(sha) == 16 and sha == bench.kernel_source_sha()


def test_cpu_baseline_reports_all_cores_and_one_thread():
    import argparse
    w = W.workload("tiny")
    args = argparse.Namespace(cpu_max_steps=3, cpu_budget_s=5.0)
    r = bench.cpu_baseline(w, args, caches=bench.host_cache(w, w.N0 + 2 + args.cpu_max_steps))
    assert r["kind"] == "oracle" and r["unit"] == bench.UNIT and r["value"] > 0
    assert r["cores"] >= 1 and r["cpu_model"]
    one = r["single_thread"]
    assert one["cores"] == 1 and one["value"] > 0 and one["ms_per_step"] > 0
