"""Pins of the oracle's gated delta update and readout against the printed matrix
form S_t = (I - beta k k^T) D_t S_{t-1} + beta k v^T (bloombook section 2) and the
properties the pages state for it."""
import numpy as np
import pytest

from oracle import stq_oracle as O

F32 = np.float32


def _unit(rng, n, d):
    x = rng.standard_normal((n, d))
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(F32)


def _literal(S_prev, k, v, decay, beta):
    """Printed form in float64 with explicit matrices."""
    d = S_prev.shape[-1]
    out = []
    for n in range(S_prev.shape[0]):
        kk = k[n].astype(np.float64)
        A = (np.eye(d) - beta[n] * np.outer(kk, kk)) @ np.diag(decay[n].astype(np.float64))
        out.append(A @ S_prev[n].astype(np.float64) + beta[n] * np.outer(kk, v[n].astype(np.float64)))
    return np.stack(out)


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_update_matches_literal_matrix_form(kind):
    rng = np.random.default_rng(1)
    n, d = 6, 128
    S = rng.standard_normal((n, d, d)).astype(F32)
    k = _unit(rng, n, d)
    v = rng.standard_normal((n, d)).astype(F32)
    beta = rng.random(n).astype(F32)
    if kind == "gdn":
        decay = np.repeat(np.exp(rng.uniform(-0.2, -0.001, n))[:, None], d, 1).astype(F32)
    else:
        decay = np.exp(rng.uniform(-0.5, -0.0005, (n, d))).astype(F32)
    got, _ = O.fp32_step(S, k, k, v, decay, beta)
    ref = _literal(S, k, v, decay, beta)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err < 2e-6, err
    # element-wise: within a few float32 ulps of the operands' scale
    assert np.max(np.abs(got - ref)) < 1e-5 * np.max(np.abs(ref))


def test_decay_acts_on_key_rows_not_columns():
    # D_t multiplies S_{t-1} from the left: row i is scaled by d_i.
    d = 8
    S = np.ones((1, d, d), F32)
    decay = np.linspace(0.1, 0.8, d).astype(F32)[None]
    k = np.zeros((1, d), F32); k[0, 0] = 1
    got, _ = O.fp32_step(S, k, k, np.zeros((1, d), F32), decay, np.zeros(1, F32))
    assert np.array_equal(got[0], np.repeat(decay[0][:, None], d, 1))


def test_beta_zero_identity_decay_is_exact_identity():
    rng = np.random.default_rng(2)
    S = rng.standard_normal((3, 128, 128)).astype(F32)
    k = _unit(rng, 3, 128)
    v = rng.standard_normal((3, 128)).astype(F32)
    got = O.delta_update(S, k, v, np.zeros(3, F32))
    assert np.array_equal(got, S)


def test_delta_property_unit_key_beta_one():
    # with |k| = 1 and beta = 1, k^T S_t = v^T: the write replaces the value bound to k
    rng = np.random.default_rng(3)
    S = rng.standard_normal((4, 128, 128)).astype(F32)
    k = _unit(rng, 4, 128)
    v = rng.standard_normal((4, 128)).astype(F32)
    got = O.delta_update(S, k, v, np.ones(4, F32))
    kS = np.einsum("ni,nij->nj", k.astype(np.float64), got.astype(np.float64))
    assert np.max(np.abs(kS - v)) < 1e-5 * (1 + np.max(np.abs(S)))


def test_transition_spectral_bound():
    # |A_t|_2 <= |D_t|_2 <= 1 when |k| <= 1, 0 <= beta <= 1, 0 <= D <= I (bloombook
    # section 2). A_t is read off the oracle by updating the identity with v = 0.
    rng = np.random.default_rng(4)
    d = 32
    for trial in range(400):
        k = rng.standard_normal(d)
        k *= rng.random() / np.linalg.norm(k)
        k = k.astype(F32)[None]
        beta = F32(rng.random())
        dec = rng.random(d).astype(F32)[None] if trial % 2 else np.full((1, d), rng.random(), F32)
        A, _ = O.fp32_step(np.eye(d, dtype=F32)[None], k, k, np.zeros((1, d), F32), dec, np.array([beta]))
        ref = (np.eye(d) - float(beta) * np.outer(k[0], k[0])) @ np.diag(dec[0].astype(np.float64))
        assert np.max(np.abs(A[0] - ref)) < 1e-6
        nA = np.linalg.norm(A[0].astype(np.float64), 2)
        nD = np.max(dec)
        assert nA <= nD * (1 + 1e-5) + 1e-6 and nD <= 1


def test_readout_of_single_association_returns_value():
    # From a zero state, one write with unit k and beta = 1 stores k v^T, and reading with
    # q returns (q . k) v: the output is the state read by the query.
    rng = np.random.default_rng(5)
    d = 128
    k = _unit(rng, 1, d)
    q = _unit(rng, 1, d)
    v = rng.standard_normal((1, d)).astype(F32)
    S, o = O.fp32_step(np.zeros((1, d, d), F32), q, k, v, np.ones((1, d), F32), np.ones(1, F32))
    expect = float(q[0].astype(np.float64) @ k[0].astype(np.float64)) * v[0]
    assert np.max(np.abs(o[0] - expect)) < 1e-6


def test_tree_sum_order_and_value():
    x = np.array([1e8, 1, -1e8, 1], F32)
    # tree: (1e8 + 1) + (-1e8 + 1) rounds to 1e8 + -1e8 = 0 in float32 (both +1 lost),
    # while a left-to-right sum gives 1: the pairing order is visible here
    assert O.tree_sum(x, 0) == F32(0)
    y = np.arange(128, dtype=F32)
    assert O.tree_sum(y, 0) == F32(127 * 128 / 2)
    z = np.random.default_rng(0).standard_normal((7, 64)).astype(F32)
    assert np.allclose(O.tree_sum(z, 1), z.astype(np.float64).sum(1), rtol=0, atol=1e-5)
