"""Pins of the oracle's offline lifetime-aware allocation (bloombook sections 3 and 4;
singularity-lens calibration paragraph): the lifetime weight against its closed form,
the allocation against brute force on tiny instances, the distortions against float64
numpy means."""
import itertools

import numpy as np
import pytest

from oracle import stq_alloc as A
from oracle import stq_oracle as O

F32 = np.float32


@pytest.mark.parametrize("ell", [-0.5, -0.2, -0.05, -1e-3, -1e-6, 0.0])
def test_lifetime_weight_is_the_geometric_series(ell):
    J = 1024
    got = A.lifetime_weight(np.array([ell]), J)[0]
    if ell == 0.0:
        assert got == J
    else:
        q = np.exp(2 * ell)
        assert got == pytest.approx((1 - q ** J) / (1 - q), rel=1e-12)
    # longer memory (l closer to 0) never weighs less
    assert A.lifetime_weight(np.array([ell - 0.01]), J)[0] < got


def _brute(L, Dm, cand, budget, n_piv):
    n = len(L)
    cost = L[:, None] * Dm
    risk = cost[:, -1]
    piv = sorted(range(n), key=lambda u: (-risk[u], u))[:n_piv]
    rest = [u for u in range(n) if u not in piv]
    best = None
    for combo in itertools.product(range(len(cand)), repeat=len(rest)):
        if sum(cand[c] for c in combo) > budget * len(rest):
            continue
        c = sum(cost[u, ci] for u, ci in zip(rest, combo))
        if best is None or c < best[0] - 1e-12 * abs(best[0]):
            best = (c, combo)
    return best, rest, piv


@pytest.mark.parametrize("seed", range(12))
def test_allocation_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = 6
    cand = [2, 4, 6, 8] if seed % 2 else [4, 6, 8]
    budget = [4.0, 5.0, 6.0, 7.0][seed % 4] if seed % 2 else [6.0, 5.5, 7.0, 4.0][seed % 4]
    L = A.lifetime_weight(rng.uniform(-0.3, -0.001, n))
    # distortion falls about 4x per extra bit, with unit-specific scale
    Dm = rng.lognormal(0, 1, (n, 1)) * 4.0 ** (-np.array(cand)[None, :]) * rng.uniform(0.8, 1.2, (n, len(cand)))
    Dm = np.sort(Dm, axis=1)[:, ::-1]
    n_piv = seed % 3
    bits = A.allocate(L, Dm, cand, budget, n_piv)
    (cbest, combo), rest, piv = _brute(L, Dm, cand, budget, n_piv)
    assert sorted(np.flatnonzero(bits == 16).tolist()) == sorted(piv)
    got = sum(L[u] * Dm[u, cand.index(int(bits[u]))] for u in rest)
    assert got == pytest.approx(cbest, rel=1e-12)
    assert sum(int(bits[u]) for u in rest) <= budget * len(rest)


def test_allocation_favours_long_lived_units():
    """Equal distortion curves: a unit with a larger lifetime weight never gets fewer
    bits (the objective weighs its distortion more)."""
    rng = np.random.default_rng(7)
    n = 40
    ell = rng.uniform(-0.3, -0.001, n)
    L = A.lifetime_weight(ell)
    Dm = np.tile(4.0 ** -np.array([2, 4, 6, 8], float), (n, 1))
    bits = A.allocate(L, Dm, [2, 4, 6, 8], 4.0, 0)
    order = np.argsort(L)
    assert np.all(np.diff(bits[order]) >= 0)
    assert bits.mean() <= 4.0


def test_pivots_are_the_riskiest_units():
    L = np.array([1.0, 5.0, 2.0, 9.0, 3.0])
    Dm = np.tile([4.0, 2.0, 1.0], (5, 1))
    Dm[2, -1] = 10.0                       # unit 2: risk 20 at the widest width
    bits = A.allocate(L, Dm, [4, 6, 8], 6.0, 2)
    assert sorted(np.flatnonzero(bits == 16).tolist()) == [2, 3]


def test_budget_limits_and_infeasible_budget():
    L = np.ones(4)
    Dm = np.tile([8.0, 4.0, 2.0, 1.0], (4, 1))
    assert np.all(A.allocate(L, Dm, [2, 4, 6, 8], 8.0, 0) == 8)
    assert np.all(A.allocate(L, Dm, [2, 4, 6, 8], 2.0, 0) == 2)
    with pytest.raises(ValueError):
        A.allocate(L, Dm, [4, 6, 8], 3.0, 0)


def test_row_sq_error_and_distortions_against_float64():
    rng = np.random.default_rng(3)
    N, H, d = 3, 2, 128
    S = rng.standard_normal((N, H, d, d)).astype(F32)
    Sh = (S + rng.standard_normal(S.shape).astype(F32) * F32(0.01)).astype(F32)
    e = A.row_sq_error(S, Sh)
    ref = ((S.astype(np.float64) - Sh) ** 2).sum(-1)
    assert np.allclose(e, ref, rtol=1e-5, atol=0)
    om = rng.lognormal(size=(H, d)).astype(F32)
    Dg = A.unit_distortion("gdn", e, om)
    assert np.allclose(Dg, (e.astype(np.float64) * om[None]).sum((0, 2)) / (N * d * d), rtol=1e-12)
    Dk = A.unit_distortion("kda", e, om)
    assert np.allclose(Dk, e.astype(np.float64).sum(0).reshape(-1) / (N * d), rtol=1e-12)
    # with omega = 1 the GDN distortion is the plain mean squared error
    assert np.allclose(A.unit_distortion("gdn", e, np.ones((H, d), F32)),
                       ((S.astype(np.float64) - Sh) ** 2).mean((0, 2, 3)), rtol=1e-5)


def test_distortion_shrinks_with_width():
    """The method's quantiser at a wider uniform width distorts less (a property of the
    code grid, checked on a warm random state)."""
    rng = np.random.default_rng(11)
    S = rng.standard_normal((2, 1, 128, 128)).astype(F32)
    om = rng.lognormal(size=(1, 128)).astype(F32)
    ds = []
    for b in (2, 4, 6, 8):
        rb = np.full((1, 128), b)
        u, r, c, piv = O.refit(S, om, rb)
        e = A.row_sq_error(S, O.dequantize(u, r, c, piv, rb))
        ds.append(A.unit_distortion("gdn", e, om)[0])
    assert ds[0] > ds[1] > ds[2] > ds[3] > 0


def _mixed_head_state(seed, H=3, N=2):
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((N, H, 128, 128)) * rng.lognormal(0, 1, (N, H, 128, 1))
         * rng.lognormal(0, 0.5, (N, H, 1, 128))).astype(F32)
    om = rng.lognormal(0, 1, (H, 128)).astype(F32)
    rb = rng.choice([2, 4, 6, 8], size=(H, 128))
    rb[0, 5] = 16                                   # a pivot row
    return S, om, rb


def test_in_head_error_at_own_width_is_the_pools_error():
    # a row's in-head error at the width it has in the pool is its reconstruction error
    # in that pool (refit, dequantise, row error: each pinned on its own)
    S, om, rb = _mixed_head_state(1)
    u, r, c, piv = O.refit(S, om, rb)
    cand = (2, 4, 6, 8)
    e = A.row_error_at_widths(S, c, om, cand)
    own = A.row_sq_error(S, O.dequantize(u, r, c, piv, rb))
    quant = rb != 16
    for k, b in enumerate(cand):
        sel = np.broadcast_to((rb == b)[None], own.shape)
        assert np.array_equal(e[..., k][sel], own[sel])
    assert quant.sum() < rb.size


def test_in_head_error_never_grows_with_width_and_stops_at_full_reach():
    S, om, rb = _mixed_head_state(2)
    _, r, c, _ = O.refit(S, om, rb)
    cand = (2, 4, 6, 8)
    e = A.row_error_at_widths(S, c, om, cand).astype(np.float64)
    assert np.all(np.diff(e, axis=-1) <= 1e-6 * e[..., :1])
    # a row none of whose codes reaches +-qmax_b at width b gains nothing from more bits:
    # the codes are rint of the same exact quotients
    rr = (A.tree_sum(np.abs(S), axis=-1) * F32(1 / 128) * O.row_gain(om)).astype(F32)
    y = (S * O._recip(rr)[..., :, None]).astype(F32)
    x = np.abs(y.astype(np.float64) * O._recip(c).astype(np.float64)[..., None, :]).max(axis=-1)
    fits = x < 31.5                                  # within reach at 6 bits
    assert fits.any()
    assert np.array_equal(e[..., 2][fits], e[..., 3][fits])


def test_in_head_error_of_a_uniform_head_matches_uniform_measure_at_its_width():
    # in a head of one width the in-head error at that width is the uniform-width
    # distortion measure the first allocation uses
    rng = np.random.default_rng(3)
    S = (rng.standard_normal((2, 2, 128, 128)) * rng.lognormal(0, 1, (2, 2, 128, 1))).astype(F32)
    om = rng.lognormal(0, 1, (2, 128)).astype(F32)
    for b in (2, 4, 6, 8):
        rb = np.full((2, 128), b)
        u, r, c, piv = O.refit(S, om, rb)
        e = A.row_error_at_widths(S, c, om, (b,))[..., 0]
        assert np.array_equal(e, A.row_sq_error(S, O.dequantize(u, r, c, piv, rb)))
