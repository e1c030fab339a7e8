"""Pins for the oracle's selector variants (max-over-heads scores, forced sink/local
blocks, per-query-head selection), each against something other than itself: special
cases that reduce to the pinned base selector, the bound property, exact dot products
when a block holds one token, and brute-force enumeration on tiny inputs."""
import itertools

import numpy as np
import pytest

import oracle as OR
import workloads as W


@pytest.fixture(scope="module")
def o():
    return OR.default()


def _grid(rng, shape):
    return W.bf16_bits_to_f32(W.f32_to_bf16_bits(rng.integers(-8, 9, size=shape).astype(np.float32) / 8)).astype(np.float64)


def _summaries(k, bs):
    n, d = k.shape
    nb = -(-n // bs)
    lo = np.stack([k[b * bs:min(n, (b + 1) * bs)].min(0) for b in range(nb)])
    hi = np.stack([k[b * bs:min(n, (b + 1) * bs)].max(0) for b in range(nb)])
    return lo, hi


def test_max_scores_reduce_to_sum_for_one_head(o):
    rng = np.random.default_rng(1)
    k = _grid(rng, (700, 64))
    lo, hi = _summaries(k, 64)
    q = _grid(rng, (1, 64))
    assert np.array_equal(o.block_scores_max(q, lo, hi), o.block_scores(q, lo, hi))


def test_max_scores_bound_and_tightness(o):
    rng = np.random.default_rng(2)
    G, d = 4, 32
    q = _grid(rng, (G, d))
    k = _grid(rng, (512, d))
    lo, hi = _summaries(k, 64)
    s = o.block_scores_max(q, lo, hi)
    true_max = np.array([max((q @ k[b * 64:(b + 1) * 64].T).max(1)) for b in range(len(s))])
    assert np.all(s >= true_max - 1e-12)  # an upper bound of every head's best q.k
    lo1, hi1 = _summaries(k[:40], 1)      # one token per block: the bound is exact
    assert np.allclose(o.block_scores_max(q, lo1, hi1), (q @ k[:40].T).max(0), atol=1e-12)


def test_forced_without_forcing_is_plain_top_k(o):
    rng = np.random.default_rng(3)
    for _ in range(20):
        v = rng.integers(0, 6, size=30).astype(np.float64)  # many ties
        assert np.array_equal(o.top_ranked_forced(v, 7, 0, 0), o.top_ranked(v, 7))


def _brute_forced(v, K, n_sink, n_local):
    nb = len(v)
    keff = min(K, nb)
    forced = []
    for b in range(min(n_sink, nb)):
        if len(forced) < keff:
            forced.append(b)
    for i in range(n_local):
        b = nb - 1 - i
        if b < 0 or len(forced) >= keff:
            break
        if b not in forced:
            forced.append(b)
    rest = [b for b in range(nb) if b not in forced]
    need = keff - len(forced)
    key = lambda b: (-v[b], b)  # (value desc, index asc)
    winners = []
    for sub in itertools.combinations(rest, need):
        others = [b for b in rest if b not in sub]
        if all(key(a) < key(b) for a in sub for b in others):
            winners.append(sub)
    assert len(winners) == 1
    return sorted(forced + list(winners[0]))


@pytest.mark.parametrize("seed", range(12))
def test_forced_matches_brute_force(o, seed):
    rng = np.random.default_rng(100 + seed)
    nb = int(rng.integers(1, 11))
    K = int(rng.integers(1, 6))
    n_sink, n_local = int(rng.integers(0, 3)), int(rng.integers(0, 3))
    v = rng.integers(0, 4, size=nb).astype(np.float64)
    assert list(o.top_ranked_forced(v, K, n_sink, n_local)) == _brute_forced(v, K, n_sink, n_local)


def test_forced_overflow_prefers_sinks_then_newest(o):
    v = np.arange(10, dtype=np.float64)  # scores favour the last blocks
    assert list(o.top_ranked_forced(v, 3, 2, 4)) == [0, 1, 9]


def test_per_head_selection_is_each_heads_own_top_k(o):
    rng = np.random.default_rng(4)
    k = _grid(rng, (900, 64))
    lo, hi = _summaries(k, 64)
    q = _grid(rng, (3, 64))
    per_head = o.select_per_head(q, lo, hi, 5)
    for h in range(3):
        assert np.array_equal(per_head[h], o.top_ranked(o.block_scores(q[h:h + 1], lo, hi), 5))
