"""The speculation-budget profiler on a B200 (marked gpu): a small grid of contexts and
budgets is timed through the two-stream step, fitted, and queried."""
import math

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, never run there
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import dynamic_sparse_attention_block_b200 as prr  # noqa: E402
from dynamic_sparse_attention_block_b200.budget import SpecBudget, profile  # noqa: E402


def test_profile_fit_choose():
    base = prr.Dims(B=1, Hq=8, Hkv=2, d=128, bs=64, cap_tokens=1, K=16, P=1)
    contexts, p_grid = [4096, 8192, 16384], [8, 16]
    prof = profile(base, contexts, p_grid, steps=4, warmup=2)
    for key in prof.select_us:
        assert 0 < prof.select_us[key] < 1e4 and math.isfinite(prof.select_us[key])
        assert 0 < prof.spec_us[key] < 1e4 and math.isfinite(prof.spec_us[key])
    model = SpecBudget.fit(prof, degree=1)
    for n in (4096, 12000, 65536):
        assert model.choose(n) in (0, 8, 16)
