"""The speculation-budget profiler on a B200 (marked gpu): a small grid of contexts and
budgets is timed through the two-stream step and through the fused step, fitted, and
queried -- inside the profiled grid and beyond it -- and the library's fit and choice
are compared with the numpy reference (oracle/budget.py) on the same profiled numbers."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, never run there
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import dynamic_sparse_attention_block_b200 as prr  # noqa: E402
from dynamic_sparse_attention_block_b200.budget import SpecBudget, profile, profile_fused  # noqa: E402
from oracle import budget as REF  # noqa: E402

CONTEXTS = [4096, 8192, 16384]
P_GRID = [8, 16]
QUERIES = [2048, 4096, 12000, 16384, 65536, 262144]  # below, inside and far beyond the grid


def check_against_reference(prof, degree):
    for key in prof.select_us:
        assert 0 < prof.select_us[key] < 1e4 and math.isfinite(prof.select_us[key])
        assert 0 < prof.spec_us[key] < 1e4 and math.isfinite(prof.spec_us[key])
    model = SpecBudget.fit(prof, degree=degree)
    ctx = [n for (n, _) in prof.select_us]
    ref_sel = REF.fit(ctx, [prof.select_us[k] for k in prof.select_us], degree)
    ref_spec = [REF.fit(prof.contexts, [prof.spec_us[(n, p)] for n in prof.contexts], degree) for p in prof.p_grid]
    scale = max(prof.select_us.values())
    assert np.allclose(model.sel_coef, ref_sel, rtol=1e-6, atol=1e-9 * scale)
    for got, ref in zip(model.spec_coef, ref_spec):
        assert np.allclose(got, ref, rtol=1e-6, atol=1e-9 * scale)
    for n in QUERIES:
        sel, spec = REF.evaluate(ref_sel, n), [REF.evaluate(c, n) for c in ref_spec]
        # a choice that rests on a near tie of the two models may go either way
        if min(abs(s - sel) for s in spec) <= 1e-6 * max(1.0, abs(sel)):
            continue
        assert model.choose(n) == REF.choose(ref_sel, ref_spec, prof.p_grid, n), n


@pytest.mark.parametrize("degree", [1, 2])
def test_profile_two_stream_matches_reference(degree):
    base = prr.Dims(B=1, Hq=8, Hkv=2, d=128, bs=64, cap_tokens=1, K=16, P=1)
    check_against_reference(profile(base, CONTEXTS, P_GRID, steps=4, warmup=2), degree)


@pytest.mark.parametrize("degree", [1, 2])
def test_profile_fused_matches_reference(degree):
    base = prr.Dims(B=1, Hq=8, Hkv=2, d=128, bs=64, cap_tokens=1, K=16, P=1)
    check_against_reference(profile_fused(base, CONTEXTS, P_GRID, steps=4, warmup=2), degree)
