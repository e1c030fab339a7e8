"""Batch sharding of the decode step on CPU: the shard partition, and two gloo ranks
(world size 2) that each run the fp64 oracle's step on their own sequences and
all-gather the outputs, which must equal the oracle's step over the whole batch.  The
method needs no exchange between shards, so this checks the host logic that a
multi-GPU run uses (the split of the batch and the optional gather of the outputs)."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import workloads as W  # noqa: E402
from dynamic_sparse_attention_block_b200.sharding import gather_outputs, shard_dims, shard_ranges  # noqa: E402
from dynamic_sparse_attention_block_b200 import Dims  # noqa: E402


def test_shard_ranges_cover_the_batch_once():
    for B in (0, 1, 5, 16):
        for world in (1, 2, 3, 8):
            r = shard_ranges(B, world)
            assert len(r) == world
            assert r[0][0] == 0 and r[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            sizes = [b1 - b0 for b0, b1 in r]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def test_shard_dims_keep_the_shape():
    d = Dims(B=10, Hq=32, Hkv=8, d=128, bs=64, cap_tokens=1000, K=8, P=8, selector="per_head", n_sink=1)
    s = shard_dims(d, (3, 7))
    assert s.B == 4 and (s.Hq, s.Hkv, s.d, s.bs, s.cap_tokens, s.K, s.P, s.selector, s.n_sink) == \
        (32, 8, 128, 64, 1000, 8, 8, "per_head", 1)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_step(w, b0, b1, steps):
    """The oracle's decode steps for sequences [b0, b1) of the workload (its own shard)."""
    import oracle as OR
    o = OR.default()
    sub = w.with_(B=b1 - b0)
    cap = w.N0 + steps
    kc = np.zeros((sub.B, w.Hkv, cap, w.d), np.uint16)
    vc = np.zeros_like(kc)
    for i, b in enumerate(range(b0, b1)):
        for h in range(w.Hkv):
            k0, v0 = W.kv_prefix(w, b, h)
            kn, vn = W.kv_appended(w, b, h, steps)
            kc[i, h, :w.N0], vc[i, h, :w.N0] = k0, v0
            kc[i, h, w.N0:], vc[i, h, w.N0:] = kn, vn
    st = OR.new_state(sub.B, w.Hkv, cap, w.bs, w.d)
    for i in range(sub.B):
        for h in range(w.Hkv):
            lo, hi = o.build_summaries(kc[i, h], w.N0, w.bs)
            st["smin"][i, h, :lo.shape[0]], st["smax"][i, h, :lo.shape[0]] = lo, hi
    qs = W.queries(w, steps)[:, b0:b1]
    dims = dict(B=sub.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, bs=w.bs, cap=cap, K=w.K, P=w.P, alpha=w.alpha, scale=w.scale())
    pred = np.full((sub.B, w.Hkv, w.P), -1, np.int32)
    pred[:, :, :w.P] = np.arange(w.P)
    for t in range(steps):
        seq = np.full(sub.B, w.N0 + t + 1, np.int32)
        r = o.decode_step(dims, qs[t], kc, vc, seq, pred, st)
        pred = r["pred_next"]
    return r


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.workload("tiny").with_(B=5, Hq=4, Hkv=2, N0=700, bs=64, K=4, P=4, per_seq_seed=True)
        ranges = shard_ranges(w.B, world)
        b0, b1 = ranges[rank]
        r = _oracle_step(w, b0, b1, steps=3)
        out = gather_outputs(torch.from_numpy(r["out"]), ranges)
        lse = gather_outputs(torch.from_numpy(r["lse"]), ranges)
        q.put((rank, out.numpy(), lse.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_shards_gather_the_whole_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (o, l)) for r, o, l in (q.get(timeout=300) for _ in range(world)))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = W.workload("tiny").with_(B=5, Hq=4, Hkv=2, N0=700, bs=64, K=4, P=4, per_seq_seed=True)
    full = _oracle_step(w, 0, w.B, steps=3)
    for r in range(world):  # every rank holds the whole batch, in sequence order
        assert np.array_equal(got[r][0], full["out"]) and np.array_equal(got[r][1], full["lse"])


class _FakeShard:
    """Stands in for PRRDecoder in the host-logic test: records the rows it is given."""

    def __init__(self, dims, dev):
        self.dims, self.given, self.calls = dims, dev, []
        self.device = -1  # torch.cuda.device(-1) is a no-op, so no GPU is touched
        self.out = torch.zeros((dims.B, dims.Hq, dims.d))
        self.lse = torch.zeros((dims.B, dims.Hq))

    def step_fused(self, q, k_new, v_new):
        self.calls.append((q.clone(), k_new.clone(), v_new.clone()))


def test_sharded_decoder_hands_each_shard_its_own_rows():
    from dynamic_sparse_attention_block_b200 import Dims
    from dynamic_sparse_attention_block_b200.sharding import ShardedDecoder
    dims = Dims(B=5, Hq=4, Hkv=2, d=64, bs=64, cap_tokens=128, K=2, P=2)
    made = []

    def make(d, dev):
        made.append(_FakeShard(d, dev))
        return made[-1]

    sh = ShardedDecoder(dims, devices=["gpu0", "gpu1", "gpu2"], make=make)  # one process, three GPUs
    assert [(f.dims.B, f.given) for f in made] == [(2, "gpu0"), (2, "gpu1"), (1, "gpu2")]
    q = torch.arange(5 * 4 * 64, dtype=torch.float32).view(5, 4, 64)
    kn = torch.arange(5 * 2 * 64, dtype=torch.float32).view(5, 2, 64)
    vn = -kn
    sh.step_fused(q, kn, vn)
    for (b0, b1), f in sh.shards:
        (gq, gk, gv), = f.calls
        assert torch.equal(gq, q[b0:b1]) and torch.equal(gk, kn[b0:b1]) and torch.equal(gv, vn[b0:b1])
    assert [rng for rng, _, _ in sh.outputs()] == [(0, 2), (2, 4), (4, 5)]

    # one process per GPU: rank 1 of 3 builds only its own shard
    made.clear()
    one = ShardedDecoder(dims, devices=["mine"], rank=1, world=3, make=make)
    assert [rng for rng, _ in one.shards] == [(2, 4)] and made[0].given == "mine"
    # a batch smaller than the world leaves empty shards out
    made.clear()
    small = ShardedDecoder(Dims(B=1, Hq=4, Hkv=2, d=64, bs=64, cap_tokens=128, K=2, P=2),
                           devices=["a", "b"], make=make)
    assert len(small.shards) == 1 and len(made) == 1
    with pytest.raises(ValueError):
        ShardedDecoder(dims, devices=["a", "b"], world=3, make=make)
