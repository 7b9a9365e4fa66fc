"""Host functions of the offline width allocation (lifetime weights, unit distortions,
budgeted allocation with FP16 pivots) against the oracle: they take no GPU, so they run
here. Both sides get the same inputs; integer decisions must agree exactly."""
import numpy as np
import pytest

from oracle import stq_alloc as A
from quantized_linear_attention_02_b200 import stq

F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from quantized_linear_attention_02_b200 import build
    build.build()
    stq.lib()


def test_lifetime_weights_match_oracle():
    rng = np.random.default_rng(0)
    ell = np.concatenate([rng.uniform(-0.5, 0, 200), [0.0, -1e-9, -2.0]])
    for J in (1, 7, 1024):
        got = stq.lifetime_weights(ell, J)
        ref = A.lifetime_weight(ell, J)
        assert np.allclose(got, ref, rtol=1e-14, atol=0)
    with pytest.raises(stq.StqError):
        stq.lifetime_weights(np.array([0.1]), 10)


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_unit_distortion_bit_exact(kind):
    rng = np.random.default_rng(1)
    N, H = 3, 5
    e = rng.lognormal(size=(N, H, 128)).astype(F32)
    om = rng.lognormal(size=(H, 128)).astype(F32)
    assert np.array_equal(stq.unit_distortion(kind, e, om), A.unit_distortion(kind, e, om))


def _instance(rng, n, cand):
    L = A.lifetime_weight(rng.uniform(-0.3, -0.0005, n))
    Dm = rng.lognormal(0, 1, (n, 1)) * 4.0 ** (-np.array(cand, float))[None] * rng.uniform(0.7, 1.3, (n, len(cand)))
    return L, np.sort(Dm, axis=1)[:, ::-1].copy()


@pytest.mark.parametrize("n,cand,budget,n_piv,seed", [
    (48, (4, 6, 8), 6.0, 1, 0), (48, (2, 4, 6, 8), 4.0, 1, 1), (4096, (4, 6, 8), 6.0, 82, 2),
    (4096, (2, 4, 6, 8), 4.0, 82, 3), (9, (2, 4, 6, 8), 5.3, 0, 4), (300, (4, 8), 6.0, 6, 5)])
def test_allocation_bit_exact(n, cand, budget, n_piv, seed):
    rng = np.random.default_rng(seed)
    L, Dm = _instance(rng, n, cand)
    got = stq.allocate_bits(L, Dm, cand, budget, n_piv)
    ref = A.allocate(L, Dm, cand, budget, n_piv)
    assert np.array_equal(got.astype(np.int64), ref)
    rest = got != 16
    assert (got == 16).sum() == n_piv and got[rest].astype(int).sum() <= budget * rest.sum()


def test_allocation_ties_and_equal_costs():
    """Equal costs everywhere: both sides keep the narrowest width and the smallest total."""
    L = np.ones(10)
    Dm = np.ones((10, 4))
    cand = (2, 4, 6, 8)
    got = stq.allocate_bits(L, Dm, cand, 6.0, 2)
    assert np.array_equal(got.astype(np.int64), A.allocate(L, Dm, cand, 6.0, 2))
    assert list(got[:2]) == [16, 16] and np.all(got[2:] == 2)


@pytest.mark.parametrize("bad", ["infeasible", "cand_order", "cand_width", "pivots"])
def test_allocation_rejects_bad_arguments(bad):
    L, Dm = np.ones(4), np.ones((4, 3))
    cand, budget, n_piv = (4, 6, 8), 6.0, 0
    if bad == "infeasible":
        budget = 3.0
    elif bad == "cand_order":
        cand = (6, 4, 8)
    elif bad == "cand_width":
        cand = (4, 5, 8)
    else:
        n_piv = 5
    with pytest.raises(stq.StqError):
        stq.allocate_bits(L, Dm, cand, budget, n_piv)
