"""Host-side logic on CPU: the seeded input generators and the bench's byte accounting.

The generators feed both the oracle and the CUDA path, so their contract (exact bf16
rounding, the forced-overlap construction, determinism) is checked on its own here.
"""
import numpy as np
import pytest

import bench
import workloads as W


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], np.float32)
    bits = W.f32_to_bf16_bits(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins; 1 + 3*2^-8 rounds up
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000]
    assert np.array_equal(W.bf16_bits_to_f32(bits), np.array([1.0, 1.0, 1.0 + 2.0 ** -6, -2.5, 0.0], np.float32))


def test_grid_values_and_determinism():
    w = W.workload("tiny")
    q1, q2 = W.queries(w, 4), W.queries(w, 4)
    assert np.array_equal(q1, q2)
    vals = W.bf16_bits_to_f32(q1).ravel() * 8
    assert np.all(vals == np.round(vals)) and vals.min() >= -8 and vals.max() <= 8
    k, v = W.kv_prefix(w, 0, 0, 256)
    kv = W.bf16_bits_to_f32(k) * 8
    assert np.all(kv == np.round(kv))
    assert np.abs(W.bf16_bits_to_f32(v)).max() < 8  # N(0,1) values, not grid


def test_query_walk_keeps_most_channels():
    w = W.workload("llama8b_32k")
    q = W.queries(w, 8)
    same = np.mean(q[1:] == q[:-1])
    # kept with probability 0.9, or redrawn to the same grid value (1/17)
    assert 0.85 < same < 0.97


@pytest.mark.parametrize("overlap,kept", [(1.0, 64), (0.97, 62), (0.9, 58), (0.75, 48), (0.5, 32), (0.0, 0)])
def test_forced_prediction_overlap(overlap, kept):
    w = W.workload("repair_sweep_64k")
    rng = np.random.default_rng(3)
    nb = 1025
    sel = np.sort(rng.choice(nb, size=64, replace=False))
    assert W.forced_kept_count(overlap, 64) == kept
    fp = W.forced_prediction(w, sel, nb, overlap, 1, 5, 2, 3)
    assert len(fp) == 64 and np.all(np.diff(fp) > 0) and fp.min() >= 0 and fp.max() < nb
    assert len(np.intersect1d(fp, sel)) == kept
    assert np.array_equal(fp, W.forced_prediction(w, sel, nb, overlap, 1, 5, 2, 3))


@pytest.mark.parametrize("name,mb", [("llama8b_32k", 18.88), ("batched_128k", 335.6), ("long_512k", 201.3)])
def test_algorithmic_bytes(name, mb):
    # summaries of every block (2d bf16 each) + K and V of the K_eff selected blocks
    w = W.workload(name)
    b = bench.algorithmic_bytes(w, w.N0 + 1)
    assert b["total"] == b["summaries"] + b["kv"]
    assert abs(b["total"] / 1e6 - mb) < 0.05 * mb


def test_batch_override_for_reduced_captures():
    class A:
        workload, batch = "batched_128k", 6
    w = bench.base_workload(A())
    assert w.B == 6 and w.N0 == W.workload("batched_128k").N0


def test_trace_summary_on_a_synthetic_timeline():
    """Records carry their item kind (1 selection chunk, 2 speculative block, 3 repair,
    4 predictor, 5 merge, 6 finisher); records that never ran stay zero and are
    ignored."""
    from dynamic_sparse_attention_block_b200.decoder import summarize_trace
    ns = 1000
    trace = np.array([[10 * ns, 14 * ns, (3 << 32) | 1, 1],
                      [11 * ns, 15 * ns, (4 << 32) | 2, 1],
                      [15 * ns, 20 * ns, (3 << 32) | (1 << 16) | 1, 3],
                      [12 * ns, 16 * ns, (5 << 32) | 3, 2],
                      [16 * ns, 19 * ns, (5 << 32) | 3, 6],
                      [0, 0, 0, 0]], np.int64)  # last record never ran
    s = summarize_trace(trace)
    assert s["sel"]["n"] == 2 and s["sel"]["start_min_us"] == 0.0 and s["sel"]["end_max_us"] == 5.0
    assert s["repair"]["dur_p50_us"] == 5.0 and s["repair"]["sms"] == 1
    assert s["spec"]["n"] == 1 and s["spec"]["start_min_us"] == 2.0
    assert s["ema"]["n"] == 0 and s["end_us"] == 10.0
    assert s["finish"]["n"] == 1 and s["finisher"] == {"n": 1, "dur_p50_us": 3.0, "dur_max_us": 3.0}


def test_rep_offsets_are_seeded_and_in_range():
    """Representative offsets (an input of the representative-key selector) depend only
    on the workload's seed, the sequence and the KV head, and lie inside a block."""
    w = W.workload("tiny").with_(selector="representative", n_rep=4, B=2, Hkv=2, Hq=8)
    a = W.rep_offsets(w, 1, 1, 70)
    assert a.shape == (70, 4) and a.dtype == np.uint8
    assert a.min() >= 0 and a.max() < w.bs
    assert np.array_equal(a, W.rep_offsets(w, 1, 1, 70))
    assert not np.array_equal(a, W.rep_offsets(w, 1, 0, 70))


# The benchmarked configurations: (B, Hq, Hkv, d, N0, bs, K, P, steps, q/k kind, walk p)
CONFIGS = {
    "tiny": (1, 4, 1, 64, 4096, 64, 8, 8, 16, "grid", 0.9),
    "llama8b_32k": (1, 32, 8, 128, 32768, 64, 64, 64, 128, "grid", 0.9),
    "batched_128k": (16, 32, 8, 128, 131072, 128, 32, 32, 64, "grid", 0.9),
    "repair_sweep_64k": (8, 32, 8, 128, 65536, 64, 64, 64, 32, "gauss", 0.9),
    "long_512k": (4, 64, 8, 128, 524288, 128, 64, 64, 32, "grid", 0.8),
}


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_workload_shapes_are_the_benchmarked_configs(name):
    w = W.workload(name)
    got = (w.B, w.Hq, w.Hkv, w.d, w.N0, w.bs, w.K, w.P, w.steps, w.qk, w.walk_p)
    assert got == CONFIGS[name]
    assert w.nb(w.N0 + 1) == -(-(w.N0 + 1) // w.bs)
    if name == "repair_sweep_64k":  # six forced predictor-overlap levels
        assert tuple(w.forced_overlaps) == (1.0, 0.97, 0.9, 0.75, 0.5, 0.0)
    if name == "batched_128k":
        assert w.per_seq_seed  # seed = b per sequence
