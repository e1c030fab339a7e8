"""Profiling-guided speculation budget on CPU: the numpy reference against closed forms,
then the library's host functions (prr_budget_fit / prr_budget_choose) and the
SpecBudget model against the reference."""
import numpy as np
import pytest

from oracle import budget as REF
from dynamic_sparse_attention_block_b200 import PrrError, _abi, build
from dynamic_sparse_attention_block_b200.budget import Profile, SpecBudget

CTX = np.array([4096, 16384, 32768, 65536, 131072, 262144, 524288], np.float64)


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build(verbose=False)
    return _abi.load()


# ----------------------------------------------------------------------------- reference pins

@pytest.mark.parametrize("degree", [0, 1, 2, 3])
def test_reference_recovers_exact_polynomials(degree):
    coef = np.array([3.0, -1.5, 0.25, 0.02])[:degree + 1]
    y = np.polynomial.polynomial.polyval(CTX / 65536.0, coef)
    assert np.allclose(REF.fit(CTX, y, degree), coef, rtol=1e-9, atol=1e-9)


def test_reference_fit_is_least_squares():
    rng = np.random.default_rng(5)
    y = 10 + 3 * CTX / 65536 + rng.normal(0, 0.5, CTX.shape)
    c = REF.fit(CTX, y, 1)
    v = np.vander(CTX / 65536, 2, increasing=True)
    assert np.allclose(v.T @ (y - v @ c), 0.0, atol=1e-8)  # residual orthogonal to the columns


def test_reference_choice_by_hand():
    # at 128K tokens (x = 2): selection 3 + 2*2 + 0.5*4 = 9 us; speculation 3.4, 6.2, 13.4 us
    sel = [3.0, 2.0, 0.5]
    spec = [[1, 1, 0.1], [2, 1.5, 0.3], [5, 3, 0.6]]
    assert REF.choose(sel, spec, [16, 32, 64], 131072) == 32
    # at 4K tokens (x = 1/16): selection 3.13 us; speculation 1.06, 2.10, 5.19 us
    assert REF.choose(sel, spec, [16, 32, 64], 4096) == 32
    assert REF.choose([20.0, 0.0, 0.0], spec, [16, 32, 64], 4096) == 64  # everything fits
    assert REF.choose([0.0, 0.0, 0.0], spec, [16, 32, 64], 131072) == 0


# ----------------------------------------------------------------------------- library vs reference

@pytest.mark.parametrize("degree", [0, 1, 2, 3])
def test_fit_matches_reference(degree):
    rng = np.random.default_rng(degree)
    y = 5 + 4 * CTX / 65536 + 0.3 * (CTX / 65536) ** 2 + rng.normal(0, 0.2, CTX.shape)
    got = _abi.prr_budget_fit(CTX, y, degree)
    ref = REF.fit(CTX, y, degree)
    assert np.allclose(got, ref, rtol=1e-8, atol=1e-8)


def test_choose_matches_reference():
    rng = np.random.default_rng(11)
    p_grid = [8, 16, 32, 64, 96]
    for _ in range(50):
        sel = rng.uniform(0, 10, 3)
        spec = rng.uniform(0, 10, (len(p_grid), 3))
        for n in (2048, 32768, 131072, 524288, 1048576):
            assert _abi.prr_budget_choose(sel, spec, p_grid, n) == REF.choose(sel, spec, p_grid, n)


def test_errors():
    with pytest.raises(PrrError) as e:
        _abi.prr_budget_fit([4096.0, 8192.0], [1.0, 2.0], 2)  # two points, three coefficients
    assert e.value.status == 2
    with pytest.raises(PrrError) as e:
        _abi.prr_budget_fit([4096.0] * 4, [1.0, 2.0, 3.0, 4.0], 1)  # one distinct context
    assert e.value.status == 1
    with pytest.raises(PrrError) as e:
        _abi.prr_budget_choose([1.0], [[0.5], [0.6]], [32, 16], 4096)  # grid not ascending
    assert e.value.status == 2


# ----------------------------------------------------------------------------- the model

def test_spec_budget_from_a_profile():
    """Selection grows linearly with context, speculation with P; the budget that fits
    under selection grows with the context."""
    contexts, p_grid = [16384, 65536, 131072, 262144], [16, 32, 64]
    sel = {(n, p): 5.0 + 10.0 * n / 65536 for n in contexts for p in p_grid}
    spec = {(n, p): 2.0 + 0.5 * p for n in contexts for p in p_grid}
    model = SpecBudget.fit(Profile(contexts, p_grid, sel, spec), degree=1)
    # selection: 5 + 10x us; speculation: 10, 18, 34 us for P = 16, 32, 64
    assert model.choose(16384) == 0      # 7.5 us of selection hides no budget
    assert model.choose(65536) == 16     # 15 us
    assert model.choose(131072) == 32    # 25 us
    assert model.choose(262144) == 64    # 45 us
    for n in (20000, 100000, 400000):
        assert model.choose(n) == REF.choose(model.sel_coef, model.spec_coef, p_grid, n)
