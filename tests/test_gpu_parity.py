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
def test_decode_append_in_step(mode):
    """The step appends its own token (k_new / v_new in the step buffers): the fused
    launch writes the row, attends it from k_new / v_new and advances seq_lens itself;
    the two-stream step launches the append first.  Same results as appending first."""
    w = W.workload("tiny").with_(name="append_in_step", B=3, Hq=12, Hkv=3, d=128, N0=2000, bs=64, K=16,
                                 P=16, steps=12, walk_p=0.8)
    _assert_ok(run_parity(w, steps=12, mode=mode, append="step"))
    w2 = w.with_(N0=1983, bs=128, K=8, P=8, steps=8)  # blocks of 128, new token mid-block
    _assert_ok(run_parity(w2, steps=8, graph=True, mode=mode, append="step"))


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


def test_decode_full_size_append_in_step():
    """The headline 128K batched workload with the token appended inside the fused
    launch (the bench's end-to-end path), graphs, sampled units."""
    _assert_ok(run_parity(W.workload("batched_128k"), steps=4, units=[(0, 0), (9, 2), (15, 7)], graph=True,
                          append="step"))


# ----------------------------------------------------------------------------- selector variants

@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("selector,n_sink,n_local", [
    ("group_max", 0, 0), ("per_head", 0, 0), ("group_sum", 2, 3), ("group_max", 1, 4), ("per_head", 1, 2),
    ("representative", 0, 0), ("representative", 1, 2),
])
def test_decode_selector_variants(mode, selector, n_sink, n_local):
    """The selector variants of the representative DSA methods (group max of the
    per-head bounds, per-query-head selection, InfLLM-style representative keys, forced
    sink and local blocks) through both step implementations, every unit, against the
    oracle's variants."""
    w = W.workload("tiny").with_(name="variant", B=2, Hq=8, Hkv=2, d=128, N0=3000, bs=64, K=12, P=12, steps=6,
                                 walk_p=0.8, selector=selector, n_sink=n_sink, n_local=n_local,
                                 n_rep=3 if selector == "representative" else 0)
    _assert_ok(run_parity(w, steps=6, mode=mode))


@pytest.mark.parametrize("paged", [False, True])
def test_decode_representative_keys_in_step(paged):
    """The representative-key selector with 128-token blocks, 4 representatives, the
    token appended inside the fused launch (a representative of the tail block may be
    the new token) and, paged, its keys read through the block table."""
    w = W.workload("tiny").with_(name="rep", B=2, Hq=8, Hkv=2, d=128, N0=5000, bs=128, K=8, P=8, steps=5,
                                 walk_p=0.8, selector="representative", n_rep=4)
    _assert_ok(run_parity(w, steps=5, append="step", paged=paged))


def test_select_topk_refuses_representative_keys():
    """prr_select_topk takes no key cache, so the representative-key selector is refused
    there (PRR_ERR_SHAPE) before anything is enqueued."""
    from dynamic_sparse_attention_block_b200._abi import PrrError
    reps = torch.zeros((1, 1, 4, 2), dtype=torch.uint8, device="cuda")
    dims = prr.Dims(B=1, Hq=4, Hkv=1, d=128, bs=64, cap_tokens=256, K=2, P=2, selector="representative", n_rep=2,
                    rep_offsets=reps.data_ptr())
    ws = torch.zeros(prr.prr_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    t = torch.zeros((1, 1, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(PrrError) as err:
        prr.prr_select_topk(dims, torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda"),
                            torch.zeros((1, 1, 4, 2, 128), dtype=torch.bfloat16, device="cuda"),
                            torch.full((1,), 200, dtype=torch.int32, device="cuda"), t, t.clone(), t.clone(),
                            torch.zeros((1, 1), dtype=torch.int32, device="cuda"),
                            torch.zeros((1, 1, 2), dtype=torch.uint8, device="cuda"), ws)
    assert err.value.status == 2


@pytest.mark.parametrize("selector", ["group_max", "per_head"])
def test_decode_selector_variants_gqa8(selector):
    """8:1 GQA at the 512K workload's head shape (reduced context), forced blocks, the
    token appended inside the fused launch, CUDA graphs."""
    w = W.workload("long_512k").with_(B=1, N0=60000, steps=4, selector=selector, n_sink=1, n_local=2)
    _assert_ok(run_parity(w, steps=4, graph=True, append="step"))


@pytest.mark.parametrize("selector,K,n_sink,n_local", [
    ("group_max", 64, 0, 0), ("per_head", 16, 0, 0), ("group_sum", 3, 2, 4), ("group_sum", 20, 5, 5),
    ("per_head", 8, 1, 1),
])
def test_select_topk_variants(selector, K, n_sink, n_local):
    """prr_select_topk under each selector, bit-exact on the grid; (K=3, 2 sinks, 4
    local) overflows the budget: sinks first, then the newest local block."""
    rng = np.random.default_rng(31)
    B, Hkv, G, d, bs, n = 2, 2, 4, 128, 64, 9000
    dims = prr.Dims(B=B, Hq=G * Hkv, Hkv=Hkv, d=d, bs=bs, cap_tokens=n + 3, K=K, P=K, selector=selector,
                    n_sink=n_sink, n_local=n_local)
    k = _rng_grid(rng, (B, Hkv, n + 3, d))
    q = _rng_grid(rng, (B, G * Hkv, d))
    o = OR.default()
    nb = -(-n // bs)
    summ_h = np.zeros((B, Hkv, dims.maxnb, 2, d), np.uint16)
    lohi = {}
    for b in range(B):
        for h in range(Hkv):
            lo, hi = o.build_summaries(k[b, h], n, bs)
            lohi[(b, h)] = (lo, hi)
            summ_h[b, h, :nb, 0] = W.f32_to_bf16_bits(lo.astype(np.float32))
            summ_h[b, h, :nb, 1] = W.f32_to_bf16_bits(hi.astype(np.float32))
    S = dims.sel_heads
    pred_h = np.full((B, S, K), -1, np.int32)
    for b in range(B):
        for s_ in range(S):
            pred_h[b, s_] = np.sort(rng.choice(nb, size=K, replace=False))
    ws = torch.zeros(prr.prr_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    seq = torch.full((B,), n, dtype=torch.int32, device="cuda")
    sel = torch.zeros((B, S, K), dtype=torch.int32, device="cuda")
    missed, nm = torch.zeros_like(sel), torch.zeros((B, S), dtype=torch.int32, device="cuda")
    keep = torch.zeros((B, S, K), dtype=torch.uint8, device="cuda")
    prr.prr_workspace_init(ws)
    prr.prr_select_topk(dims, to_dev_bits(q), to_dev_bits(summ_h), seq, torch.from_numpy(pred_h).cuda(), sel, missed,
                        nm, keep, ws)
    torch.cuda.synchronize()
    assert prr.prr_get_device_status(ws) == 0
    g_sel, g_missed, g_keep = sel.cpu().numpy(), missed.cpu().numpy(), keep.cpu().numpy()
    for b in range(B):
        for s_ in range(S):
            kvh, rows = (s_ // G, slice(s_, s_ + 1)) if selector == "per_head" else (s_, slice(s_ * G, (s_ + 1) * G))
            lo, hi = lohi[(b, kvh)]
            qg = f64(q[b, rows])
            sc = o.block_scores_max(qg, lo, hi) if selector == "group_max" else o.block_scores(qg, lo, hi)
            ref = o.top_ranked_forced(sc, K, n_sink, n_local) if (n_sink or n_local) else o.top_ranked(sc, K)
            assert np.array_equal(g_sel[b, s_], pad(ref, K)), (b, s_, g_sel[b, s_].tolist(), ref.tolist())
            ref_missed, ref_keep = o.missed_keep(ref, pred_h[b, s_])
            assert np.array_equal(g_missed[b, s_], pad(ref_missed, K))
            assert np.array_equal(g_keep[b, s_], ref_keep)
    if (n_sink, n_local, K) == (2, 4, 3):
        assert all(list(g_sel[b, s_]) == [0, 1, nb - 1] for b in range(B) for s_ in range(S))


# ----------------------------------------------------------------------------- paged KV

@pytest.mark.parametrize("mode", MODES)
def test_decode_paged_ragged(mode):
    """Paged KV cache (every block in its own page, pages in shuffled order behind a
    block table) with a ragged batch; then 128-token pages with the token appended
    inside the step and CUDA graphs."""
    w = W.workload("tiny").with_(name="paged", B=3, Hq=8, Hkv=2, d=128, N0=2600, bs=64, K=16, P=16, steps=10,
                                 walk_p=0.8, n0_seq=(2600, 1777, 2049))
    _assert_ok(run_parity(w, steps=10, mode=mode, paged=True))
    w2 = w.with_(bs=128, n0_seq=(2600, 901, 1280))
    _assert_ok(run_parity(w2, steps=6, mode=mode, paged=True, append="step", graph=True))


def test_decode_paged_variants():
    """Paged KV under per-head selection with forced blocks (fused step)."""
    w = W.workload("tiny").with_(name="paged_variant", B=2, Hq=8, Hkv=2, d=64, N0=3000, bs=64, K=12, P=12,
                                 steps=5, walk_p=0.8, selector="per_head", n_sink=1, n_local=1, n0_seq=(3000, 2222))
    _assert_ok(run_parity(w, steps=5, paged=True))


def test_decode_paged_full_size():
    """The headline 128K batched workload on a paged cache, sampled units, graphs."""
    _assert_ok(run_parity(W.workload("batched_128k"), steps=3, units=[(0, 0), (15, 7)], graph=True, paged=True))


def test_bad_block_table_sets_status_without_fault():
    """A block-table entry outside the pool is reported (PRR_DEV_BAD_RANGE) and not read:
    the tail block's entry, which the step reads to fold the newest key."""
    w = W.workload("tiny").with_(name="paged_bad", B=1, Hq=4, Hkv=1, d=64, N0=1000, bs=64, K=4, P=4, steps=2)
    dec, dims = make_decoder(w, 2, paged=True)
    dec.block_table[0, (w.N0 - 1) // w.bs] = dims.pages + 5  # past the pool
    dec.step_fused(to_dev_bits(W.queries(w, 1)[0]))
    torch.cuda.synchronize()
    assert dec.device_status() == 5


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


def test_wait_timeout_returns_status_without_fault():
    """A bounded wait that runs out, without a fault: the workspace test word makes the
    fused step skip its selection chunks, so no unit's top-K completes and the launch's
    end-of-step wait gives up after its one-second limit with PRR_DEV_WAIT_TIMEOUT (4).
    The context stays usable: after re-initialising the workspace a normal step
    selects the oracle's top-K and matches its attention."""
    from tests.prr_harness import UnitOracle, compare_attention, Report
    w = W.workload("tiny")
    dec, dims = make_decoder(w, 4)
    dec.ws.view(torch.int32)[prr.WS_TEST_SKIP_SELECTION_OFFSET // 4] = 1
    q = W.queries(w, 1)
    dec.step_fused(to_dev_bits(q[0]))
    torch.cuda.synchronize()
    assert dec.device_status() == 4
    prr.prr_workspace_init(dec.ws)
    dec.step_fused(to_dev_bits(q[0]))
    torch.cuda.synchronize()
    assert dec.device_status() == 0
    uo = UnitOracle.create(w, 0, 0, 1, OR.default())
    n, nb, qg, s, sel = uo.select(-1, q[0])  # no token appended: n = N0
    assert np.array_equal(dec.sel[0, 0].cpu().numpy(), pad(sel, w.K))
    res = uo.finish(n, nb, qg, sel, np.zeros(0, np.int32))
    rep = Report()
    compare_attention(rep, "after timeout", dec.out[0].cpu().numpy(), dec.lse[0].cpu().numpy(), res["out"], res["lse"])
    assert not rep.messages, rep.messages


def test_sharded_decoder_matches_one_decoder():
    """Two shards of one batch (here both on cuda:0, as independent decoders that never
    wait on each other) give the same outputs, bit for bit, as one decoder over the
    whole batch: units are independent, so sharding needs no exchange."""
    from dynamic_sparse_attention_block_b200.sharding import ShardedDecoder
    w = W.workload("tiny").with_(name="shards", B=5, Hq=8, Hkv=2, d=128, N0=2000, bs=64, K=8, P=8, per_seq_seed=True)
    steps = 4
    one, dims = make_decoder(w, steps)
    dev = torch.device("cuda", 0)
    sh = ShardedDecoder(dims, [dev, dev])
    for (b0, b1), dec in sh.shards:
        for i, b in enumerate(range(b0, b1)):
            for h in range(w.Hkv):
                k0, v0 = W.kv_prefix(w, b, h)
                dec.load_context(i, h, to_dev_bits(k0), to_dev_bits(v0))
        dec.prefill(None, None, w.N0)
    kn, vn = __import__("tests.gpu_runner", fromlist=["appended_tokens"]).appended_tokens(w, steps)
    qs = W.queries(w, steps)
    for t in range(steps):
        q, k, v = to_dev_bits(qs[t]), to_dev_bits(kn[t]), to_dev_bits(vn[t])
        one.step_fused(q, k_new=k, v_new=v)
        sh.step_fused(q, k, v)
        torch.cuda.synchronize()
        for (b0, b1), out, lse in sh.outputs():
            assert torch.equal(out, one.out[b0:b1]) and torch.equal(lse, one.lse[b0:b1]), (t, b0)
    assert one.device_status() == 0 and all(d.device_status() == 0 for _, d in sh.shards)


@pytest.mark.parametrize("paged", [False, True])
def test_checkpoint_resume_bit_identical(paged):
    """Resume: n steps, the decoder's state copied to the host and loaded into a fresh
    decoder, m more steps -- bit-identical to n + m steps without the break (outputs,
    selections, EMA state and predictions)."""
    from tests.gpu_runner import appended_tokens
    w = W.workload("tiny").with_(name="resume", B=2, Hq=8, Hkv=2, d=128, N0=3000, bs=64, K=12, P=12, steps=8,
                                 walk_p=0.7, per_seq_seed=True)
    n, m = 5, 3
    kn, vn = appended_tokens(w, n + m)
    qs = W.queries(w, n + m)

    def run(dec, t0, t1):
        for t in range(t0, t1):
            dec.step_fused(to_dev_bits(qs[t]), k_new=to_dev_bits(kn[t]), v_new=to_dev_bits(vn[t]))
        torch.cuda.synchronize()

    a, _ = make_decoder(w, n + m, paged=paged)
    run(a, 0, n + m)
    b, _ = make_decoder(w, n + m, paged=paged)
    run(b, 0, n)
    ck = b.checkpoint()
    del b
    c, _ = make_decoder(w, n + m, paged=paged)
    c.restore(ck)
    run(c, n, n + m)
    for name in ("out", "lse", "sel", "missed", "ema", "seq_lens", "summ"):
        assert torch.equal(getattr(a, name), getattr(c, name)), name
    assert torch.equal(a.pred, c.pred)
    assert a.device_status() == 0 and c.device_status() == 0


def test_bad_pred_sets_status_without_fault():
    w = W.workload("tiny")
    dec, dims = make_decoder(w, 4)
    dec.pred.fill_(10**6)  # out of range: slots inactive, status set
    dec.step(to_dev_bits(W.queries(w, 1)[0]))
    torch.cuda.synchronize()
    assert dec.device_status() == 2


def test_shape_ceilings_are_refused_before_launch():
    """Dims beyond a kernel's shared-memory ceiling (include/prr.h: the selection
    finisher up to 19,715 blocks at d = 128, the predictor up to 26,890, the fused step
    up to 26,760) are refused with PRR_ERR_SHAPE before anything is enqueued; below them
    both paths run."""
    from dynamic_sparse_attention_block_b200._abi import PrrError
    bs = 64
    # maxnb: (two-stream runs, fused runs)
    for maxnb, streams_ok, fused_ok in ((19000, True, True), (24000, False, True), (28000, False, False)):
        dims = prr.Dims(B=1, Hq=4, Hkv=1, d=128, bs=bs, cap_tokens=maxnb * bs, K=8, P=8)
        dec = prr.PRRDecoder(dims)
        dec.seq_lens.fill_(4096)
        q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
        for run, ok in ((lambda: dec.step(q), streams_ok), (lambda: dec.step_fused(q), fused_ok)):
            if ok:
                run()
                torch.cuda.synchronize()
                assert dec.device_status() == 0
            else:
                with pytest.raises(PrrError) as err:
                    run()
                assert err.value.status == 2, maxnb  # PRR_ERR_SHAPE
        del dec
