"""CUDA path against the fp64 oracle, through the C ABI (needs a B200; marked gpu).

Selected / missed / predicted sets and the EMA state are compared bit-exactly; the
attention output within max-abs 2e-3 and the LSE within 1e-4 relative.
"""
import math

import numpy as np
import pytest

import oracle as OR
import workloads as W
from tests.prr_harness import OUT_TOL, LSE_RTOL, accepted_selection, f64, pad

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, never run there
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import dynamic_sparse_attention_block_b200 as prr  # noqa: E402
from tests.gpu_runner import make_decoder, run_parity, to_dev_bits  # noqa: E402


def _rng_grid(rng, shape):
    return W.f32_to_bf16_bits(rng.integers(-8, 9, size=shape).astype(np.float32) / 8)


def _rng_gauss(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


def _state(B, Hq, Hkv, d, bs, cap, K, P, n, rng, gauss=False):
    """Random caches and summaries (built by the GPU call under test or by the oracle)."""
    dims = prr.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, bs=bs, cap_tokens=cap, K=K, P=P)
    draw = _rng_gauss if gauss else _rng_grid
    k = draw(rng, (B, Hkv, cap, d))
    v = _rng_gauss(rng, (B, Hkv, cap, d))
    q = draw(rng, (B, Hq, d))
    ws = torch.zeros(prr.prr_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    return dims, k, v, q, ws


# ----------------------------------------------------------------------------- a1 summaries

@pytest.mark.parametrize("d,bs,n,begin", [(128, 64, 1000, 0), (64, 128, 300, 0), (128, 128, 777, 250)])
def test_update_summaries_exact(d, bs, n, begin):
    rng = np.random.default_rng(10)
    B, Hkv, cap = 2, 3, 1024
    dims, k, v, q, ws = _state(B, 4 * Hkv, Hkv, d, bs, cap, 8, 8, n, rng, gauss=True)
    k_dev = to_dev_bits(k)
    maxnb = dims.maxnb
    summ = torch.zeros((B, Hkv, maxnb, 2, d), dtype=torch.bfloat16, device="cuda")
    o = OR.default()
    if begin > 0:  # first build [0, begin), then fold in [begin, n)
        z = torch.zeros(B, dtype=torch.int32, device="cuda")
        e = torch.full((B,), begin, dtype=torch.int32, device="cuda")
        prr.prr_update_summaries(dims, k_dev, z, e, None, begin, summ, ws)
    tb = torch.full((B,), begin, dtype=torch.int32, device="cuda")
    te = torch.full((B,), n, dtype=torch.int32, device="cuda")
    prr.prr_update_summaries(dims, k_dev, tb, te, None, n - begin, summ, ws)
    torch.cuda.synchronize()
    assert prr.prr_get_device_status(ws) == 0
    got = summ.view(torch.int16).cpu().numpy().view(np.uint16)
    nb = -(-n // bs)
    for b in range(B):
        for h in range(Hkv):
            lo, hi = o.build_summaries(k[b, h], n, bs)
            assert np.array_equal(f64(got[b, h, :nb, 0]), lo)
            assert np.array_equal(f64(got[b, h, :nb, 1]), hi)


# ----------------------------------------------------------------------------- a2-a3 select

@pytest.mark.parametrize("d,bs,G,K,P,n,gauss", [
    (128, 64, 4, 64, 64, 32769, False),   # Llama-8B-shaped, ragged tail
    (64, 64, 4, 8, 8, 4097, False),       # tiny
    (128, 128, 8, 64, 64, 70000, False),  # 8:1 GQA
    (128, 128, 4, 32, 32, 9000, False),
    (128, 64, 4, 100, 20, 20000, False),  # K not a multiple of 32, P < K
    (128, 64, 1, 7, 0, 500, False),       # no speculation, G = 1
    (128, 64, 4, 64, 64, 3000, True),     # Gaussian
    (64, 128, 2, 128, 128, 100, False),   # K > nb
])
def test_select_topk(d, bs, G, K, P, n, gauss):
    rng = np.random.default_rng(11)
    B, Hkv = 2, 2
    cap = n + 5
    dims, k, v, q, ws = _state(B, G * Hkv, Hkv, d, bs, cap, K, P, n, rng, gauss)
    o = OR.default()
    nb = -(-n // bs)
    maxnb = dims.maxnb
    summ_h = np.zeros((B, Hkv, maxnb, 2, d), np.uint16)
    scores = {}
    for b in range(B):
        for h in range(Hkv):
            lo, hi = o.build_summaries(k[b, h], n, bs)
            summ_h[b, h, :nb, 0] = W.f32_to_bf16_bits(lo.astype(np.float32))
            summ_h[b, h, :nb, 1] = W.f32_to_bf16_bits(hi.astype(np.float32))
            scores[(b, h)] = o.block_scores(f64(q[b, h * G:(h + 1) * G]), lo, hi)
    pred_h = np.full((B, Hkv, max(P, 1)), -1, np.int32)
    for b in range(B):
        for h in range(Hkv):
            cnt = min(P, nb)
            pred_h[b, h, :cnt] = np.sort(rng.choice(nb, size=cnt, replace=False))
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    sel = torch.zeros((B, Hkv, K), dtype=torch.int32, device="cuda")
    missed = torch.zeros_like(sel)
    nm = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    keep = torch.zeros((B, Hkv, max(P, 1)), dtype=torch.uint8, device="cuda")
    pred = torch.from_numpy(pred_h).cuda()
    prr.prr_workspace_init(ws)
    near_ties = 0
    for rep in range(2):  # second call checks that the tickets re-armed
        prr.prr_select_topk(dims, to_dev_bits(q), to_dev_bits(summ_h), seq, pred, sel, missed, nm, keep, ws)
        torch.cuda.synchronize()
        assert prr.prr_get_device_status(ws) == 0
        g_sel, g_missed, g_nm, g_keep = (x.cpu().numpy() for x in (sel, missed, nm, keep))
        for b in range(B):
            for h in range(Hkv):
                s = scores[(b, h)]
                # Gaussian near ties: the GPU's set, if valid under the score gap, is the
                # one missed and keep are checked against
                ref = accepted_selection(g_sel[b, h], o.top_ranked(s, K), s, gauss)
                assert ref is not None, (b, h, g_sel[b, h].tolist())
                near_ties += int(not np.array_equal(ref, o.top_ranked(s, K)))
                assert np.array_equal(g_sel[b, h], pad(ref, K)), (b, h)
                pr = pred_h[b, h][pred_h[b, h] >= 0]
                ref_missed, ref_keep = o.missed_keep(ref, pr)
                assert np.array_equal(g_missed[b, h], pad(ref_missed, K))
                assert g_nm[b, h] == len(ref_missed)
                if P > 0:
                    assert np.array_equal(g_keep[b, h][:len(pr)], ref_keep)
    assert near_ties <= 1, f"{near_ties} near-tie selections in {2 * B * Hkv} unit-calls"


# ----------------------------------------------------------------------------- a4 EMA

@pytest.mark.parametrize("P,alpha,nb", [(64, 0.9, 513), (8, 0.9, 65), (32, 0.5, 4097), (100, 0.75, 300)])
def test_ema_predict_bit_exact(P, alpha, nb):
    rng = np.random.default_rng(12)
    B, Hkv, bs = 2, 3, 64
    K = 64
    n = nb * bs - 5
    dims = prr.Dims(B=B, Hq=Hkv, Hkv=Hkv, d=128, bs=bs, cap_tokens=n + 10, K=K, P=P, alpha=alpha)
    ws = torch.zeros(prr.prr_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    ema = torch.zeros((B, Hkv, dims.maxnb), dtype=torch.float64, device="cuda")
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    pn = torch.zeros((B, Hkv, P), dtype=torch.int32, device="cuda")
    o = OR.default()
    e_ref = np.zeros((B, Hkv, dims.maxnb))
    prr.prr_ema_predict(dims, ema, None, seq, pn, ws)
    torch.cuda.synchronize()
    assert np.array_equal(pn.cpu().numpy()[0, 0], pad(list(range(min(P, nb))), P))
    perm = rng.permutation(nb)
    for t in range(12):
        sel_h = np.full((B, Hkv, K), -1, np.int32)
        cnt = min(K, nb)
        for b in range(B):
            for h in range(Hkv):
                # temporal locality: a stable core of blocks, a random set every third step
                chosen = perm[:cnt] if t % 3 else rng.choice(nb, size=cnt, replace=False)
                sel_h[b, h, :cnt] = np.sort(chosen)
        prr.prr_ema_predict(dims, ema, torch.from_numpy(sel_h).cuda(), seq, pn, ws)
        torch.cuda.synchronize()
        g_e, g_p = ema.cpu().numpy(), pn.cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                sl = sel_h[b, h][sel_h[b, h] >= 0]
                e_ref[b, h] = o.ema_update(e_ref[b, h], nb, sl, alpha)
                assert np.array_equal(g_e[b, h], e_ref[b, h]), (t, b, h)
                assert np.array_equal(g_p[b, h], pad(o.top_ranked(e_ref[b, h, :nb], P), P)), (t, b, h)
    assert prr.prr_get_device_status(ws) == 0


# ----------------------------------------------------------------------------- a5-a6 attention

@pytest.mark.parametrize("d,bs,G,n,scheme", [
    (128, 64, 4, 5000, "random"), (128, 64, 4, 5000, "perfect"), (128, 64, 4, 5000, "adversarial"),
    (128, 128, 8, 9001, "random"), (64, 64, 4, 4097, "random"), (64, 128, 2, 7000, "partial"),
    (128, 64, 3, 3333, "empty"),
])
def test_speculate_repair_merge(d, bs, G, n, scheme):
    """Standalone speculate -> select -> repair_merge equals attention over exactly the
    selected tokens, whatever the predicted set (the invariance PRR guarantees)."""
    rng = np.random.default_rng(13)
    B, Hkv, K = 2, 2, 12
    P = 0 if scheme == "empty" else K
    cap = n + 3
    dims, k, v, q, ws = _state(B, G * Hkv, Hkv, d, bs, cap, K, P, n, rng, gauss=True)
    o = OR.default()
    nb = -(-n // bs)
    k_dev, v_dev, q_dev = to_dev_bits(k), to_dev_bits(v), to_dev_bits(q)
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    summ = torch.zeros((B, Hkv, dims.maxnb, 2, d), dtype=torch.bfloat16, device="cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    prr.prr_update_summaries(dims, k_dev, z, seq, None, n, summ, ws)
    # oracle selection on oracle summaries
    ref_sel = {}
    for b in range(B):
        for h in range(Hkv):
            lo, hi = o.build_summaries(k[b, h], n, bs)
            ref_sel[(b, h)] = o.top_ranked(o.block_scores(f64(q[b, h * G:(h + 1) * G]), lo, hi), K)
    pred_h = np.full((B, Hkv, max(P, 1)), -1, np.int32)
    for (b, h), sel in ref_sel.items():
        outside = np.setdiff1d(np.arange(nb), sel)
        if scheme == "random":
            pr = np.sort(rng.choice(nb, size=P, replace=False))
        elif scheme == "perfect":
            pr = sel
        elif scheme == "adversarial":
            pr = np.sort(rng.choice(outside, size=P, replace=False))
        elif scheme == "partial":
            pr = np.sort(np.concatenate([sel[:P // 2], rng.choice(outside, size=P - P // 2, replace=False)]))
        else:
            pr = np.zeros(0, np.int32)
        pred_h[b, h, :len(pr)] = pr
    pred = torch.from_numpy(pred_h).cuda()
    Pa = max(P, 1)
    pm = torch.zeros((B, G * Hkv, Pa), dtype=torch.float32, device="cuda")
    pl = torch.zeros_like(pm)
    pO = torch.zeros((B, G * Hkv, Pa, d), dtype=torch.float32, device="cuda")
    sel = torch.zeros((B, Hkv, K), dtype=torch.int32, device="cuda")
    missed, nm = torch.zeros_like(sel), torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    keep = torch.zeros((B, Hkv, Pa), dtype=torch.uint8, device="cuda")
    out = torch.zeros((B, G * Hkv, d), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, G * Hkv), dtype=torch.float32, device="cuda")
    prr.prr_workspace_init(ws)
    for it in range(2):
        prr.prr_speculate(dims, q_dev, k_dev, v_dev, seq, pred, pm, pl, pO, ws)
        prr.prr_select_topk(dims, q_dev, summ, seq, pred, sel, missed, nm, keep, ws)
        prr.prr_repair_merge(dims, q_dev, k_dev, v_dev, seq, missed, nm, keep, pred, pm, pl, pO, out, lse, ws)
        torch.cuda.synchronize()
        assert prr.prr_get_device_status(ws) == 0
        g_out, g_lse, g_sel = out.cpu().numpy(), lse.cpu().numpy(), sel.cpu().numpy()
        for (b, h), rs in ref_sel.items():
            assert np.array_equal(g_sel[b, h], pad(rs, K))
            for g in range(G):
                ro, rl = o.attend_blocks(f64(q[b, h * G + g]), k[b, h], v[b, h], n, bs, rs, dims.c().scale)
                assert np.max(np.abs(g_out[b, h * G + g] - ro)) <= OUT_TOL
                assert abs(g_lse[b, h * G + g] - rl) <= LSE_RTOL * abs(rl)
        # speculative partials themselves: normalised numerator and block log-sum-exp
        g_pm, g_pl, g_pO = pm.cpu().numpy(), pl.cpu().numpy(), pO.cpu().numpy()
        for (b, h) in ref_sel:
            pr = pred_h[b, h][pred_h[b, h] >= 0]
            for j, blk in enumerate(pr[:4]):
                for g in range(G):
                    m, l, O = o.block_partial(f64(q[b, h * G + g]), k[b, h], v[b, h], n, bs, int(blk), dims.c().scale)
                    row = h * G + g
                    got_lse = g_pm[b, row, j] * math.log(2.0) + math.log(g_pl[b, row, j])
                    assert abs(got_lse - (m + math.log(l))) <= LSE_RTOL * max(1.0, abs(m + math.log(l)))
                    assert np.max(np.abs(g_pO[b, row, j] / g_pl[b, row, j] - O / l)) <= OUT_TOL


# ----------------------------------------------------------------------------- full decode steps

def _assert_ok(rep):
    assert not rep.messages, "\n".join(rep.messages[:20])
    assert rep.units_compared > 0
    assert rep.max_out_err <= OUT_TOL and rep.max_lse_rel <= LSE_RTOL


MODES = ("fused", "streams")


@pytest.mark.parametrize("mode", MODES)
def test_decode_tiny_all_steps(mode):
    """Tiny workload (1 KV head x 4 query heads, d 64, 4096 tokens, 16 steps), every step."""
    _assert_ok(run_parity(W.workload("tiny"), steps=16, mode=mode))


@pytest.mark.parametrize("mode", MODES)
def test_decode_tiny_graph_replay(mode):
    """Same trajectory with the step captured once per parity in a CUDA graph."""
    _assert_ok(run_parity(W.workload("tiny"), steps=8, graph=True, mode=mode))


@pytest.mark.parametrize("mode", MODES)
def test_decode_llama8b_32k(mode):
    """Llama-3.1-8B-shaped layer at 32K (bench workload), all 8 KV heads, 12 steps, graphs."""
    _assert_ok(run_parity(W.workload("llama8b_32k"), steps=12, graph=True, mode=mode))


@pytest.mark.parametrize("mode", MODES)
def test_decode_ragged_small(mode):
    """Small ragged shapes: context not a multiple of the block, K > some nb, G = 2."""
    w = W.workload("tiny").with_(name="ragged", B=3, Hq=6, Hkv=3, d=128, N0=1000, bs=64, K=20,
                                 P=12, steps=40, walk_p=0.7)
    _assert_ok(run_parity(w, steps=40, mode=mode))
    w2 = w.with_(N0=130, bs=128, K=8, P=8, steps=5)  # K > nb for the first steps
    _assert_ok(run_parity(w2, steps=5, mode=mode))


@pytest.mark.parametrize("mode", MODES)
def test_decode_no_speculation(mode):
    """Budget P = 0: every selected block is repaired; the predictor is idle."""
    w = W.workload("tiny").with_(name="no_spec", B=2, Hq=8, Hkv=2, d=128, N0=3000, bs=64, K=16,
                                 P=0, steps=6)
    _assert_ok(run_parity(w, steps=6, mode=mode))


@pytest.mark.parametrize("mode", MODES)
def test_decode_repair_sweep_small(mode):
    """Gaussian q/k/v with forced predictor overlap at every level (reduced context)."""
    w = W.workload("repair_sweep_64k").with_(B=2, N0=8192)
    for level, ov in enumerate(w.forced_overlaps):
        _assert_ok(run_parity(w, steps=3, forced=(ov, level), mode=mode))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("d,bs,G,K,P", [
    (64, 64, 8, 128, 128),    # largest K and P (below nb), 8:1 GQA, small head dim
    (64, 128, 8, 128, 128),   # the same with large blocks: K and P above nb (take all)
    (128, 64, 1, 1, 1),       # smallest K and P, no grouping
    (64, 64, 3, 33, 17),      # odd group size, K and P not multiples of 32
    (128, 128, 5, 100, 128),  # P > K
])
def test_decode_shape_limits(mode, d, bs, G, K, P):
    """Shapes at the limits the ABI accepts (d in {64, 128}, bs in {64, 128}, G <= 8,
    K and P up to 128), several steps, all units, both step implementations."""
    w = W.workload("tiny").with_(name="limits", B=2, Hq=2 * G, Hkv=2, d=d, N0=9000 + 37, bs=bs, K=K,
                                 P=P, steps=4, walk_p=0.8)
    _assert_ok(run_parity(w, steps=4, mode=mode))


@pytest.mark.parametrize("name,steps,units", [
    ("batched_128k", 3, [(0, 0), (7, 3), (15, 7)]),
    ("long_512k", 3, [(0, 0), (2, 5), (3, 7)]),
])
def test_decode_full_size_sampled(name, steps, units):
    """Full-size workloads, the whole batch on the GPU (fused step, graphs), sampled
    units in the oracle."""
    _assert_ok(run_parity(W.workload(name), steps=steps, units=units, graph=False))


def test_decode_repair_sweep_full_size():
    """The 64K Gaussian repair sweep at full size, two overlap levels, all units."""
    w = W.workload("repair_sweep_64k")
    for level in (1, 5):  # 97% and 0% overlap
        _assert_ok(run_parity(w, steps=2, forced=(w.forced_overlaps[level], level)))


# ----------------------------------------------------------------------------- device status

def test_bad_seq_len_sets_status_without_fault():
    w = W.workload("tiny")
    dec, dims = make_decoder(w, 4)
    dec.seq_lens.fill_(dims.cap_tokens + 7)  # beyond the cache
    dec.step(to_dev_bits(W.queries(w, 1)[0]))
    torch.cuda.synchronize()
    assert dec.device_status() in (1, 5)  # bad seq_len or bad summary range, first wins
    # the context is still usable: re-initialise and run a valid step
    prr.prr_workspace_init(dec.ws)
    dec.seq_lens.fill_(w.N0)
    dec.step(to_dev_bits(W.queries(w, 1)[0]))
    torch.cuda.synchronize()
    assert dec.device_status() == 0


def test_bad_pred_sets_status_without_fault():
    w = W.workload("tiny")
    dec, dims = make_decoder(w, 4)
    dec.pred.fill_(10**6)  # out of range: slots inactive, status set
    dec.step(to_dev_bits(W.queries(w, 1)[0]))
    torch.cuda.synchronize()
    assert dec.device_status() == 2
