"""The multi-GPU bench path on CPU: two gloo ranks (world size 2).

Under torchrun each rank runs an independent replica of the decode step on its own
sequences (the path shards by (sequence, KV head) with no exchange), so the only
cross-rank logic is the whole-job reduction of the timing, the per-rank workload
seeds and the reference arm's rank handling.  All of it is host code, tested here.
"""
import argparse
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402
import workloads as W  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q, with_e2e):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tokens = 1000.0 * (rank + 1)
        secs = 0.5 + rank
        e2e = 10.0 * (rank + 1) if with_e2e else None
        out_q.put((rank, bench.reduce_over_ranks(tokens, secs, e2e, world, "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("with_e2e", [True, False])
def test_reduce_over_two_gloo_ranks(with_e2e):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = 2
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, with_e2e)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        tokens, secs, e2e = got[r]
        assert tokens == 3000.0  # sum over ranks
        assert secs == 1.5       # max over ranks
        assert e2e == (30.0 if with_e2e else None)


def test_single_rank_reduction_is_identity():
    assert bench.reduce_over_ranks(7.0, 0.25, None, 1, "cpu") == (7.0, 0.25, None)


def test_ranks_get_distinct_sequences():
    w = W.workload("tiny")
    w0, w1 = bench.rank_workload(w, 0), bench.rank_workload(w, 1)
    assert w0 == w and w1.seed != w0.seed
    assert (W.queries(w0, 2) != W.queries(w1, 2)).any()
    k0, _ = W.kv_prefix(w0, 0, 0, 64)
    k1, _ = W.kv_prefix(w1, 0, 0, 64)
    assert (k0 != k1).any()


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(workload="tiny", warmup=3, steps=2, gpus=2, ref_budget_s=1.0)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line_carries_the_gpu_arm_config(monkeypatch, capsys):
    """The reference arm prints one JSON line with the same metric, unit, direction and
    config as the GPU arm, so the two lines compare like for like."""
    import json
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    args = argparse.Namespace(workload="tiny", warmup=3, steps=2, gpus=1, ref_budget_s=5.0, batch=0)
    assert bench.run_reference(args) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(bench.base_workload(args), args)
    assert (line["metric"], line["unit"], line["higher_is_better"]) == (bench.METRIC, bench.UNIT, True)
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["value"] > 0 and line["steps"] >= 1
