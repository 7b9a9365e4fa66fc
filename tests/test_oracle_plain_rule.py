"""Pins of the plain float64 restatement of the decode step (oracle/plain_rule.py), and
how far the float32 oracle's fixed evaluation order sits from it.

The float32 oracle (`stq_oracle`) follows one evaluation order for every sum, because
codes are compared bit for bit with the GPU. `plain_rule` evaluates the same rule in
float64 with plain sums, S itself in the least-squares sums and the decay applied as a
matrix. The last test here runs both on warmed-up states of the GDN and KDA parity
workloads from one packed state and records the distance: row scales and readouts
agree to float32 rounding; the codes differ where float32 rounding moves an element
across a rounding boundary, and in the columns whose least-squares steps such a
difference changed."""
import numpy as np
import pytest

from oracle import plain_rule as P
from oracle import stq_oracle as O
from quantized_linear_attention_02_b200 import workload as W

import stq_testlib as T
from test_oracle_refit import G8, OMEGA8, _exact_refit

F32 = np.float32
D = 128


@pytest.mark.parametrize("seed,bits", [
    (0, [8] * 8), (1, [6] * 8), (2, [4] * 8), (3, [2] * 8),
    (4, [2, 4, 6, 8, 16, 8, 6, 4]), (5, [6, 16, 6, 6, 4, 8, 16, 2]),
])
def test_plain_refit_matches_exact_rational_rule(seed, bits):
    # exact rationals (tests/test_oracle_refit.py) evaluate num_j with y = S / r; the
    # plain rule with S (omega r Q S = omega r^2 Q y exactly)
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((8, 8)) * rng.lognormal(0, 1, (8, 1)) * rng.lognormal(0, 1, (1, 8))).astype(F32)
    Q, r, c, piv = P.refit(S, OMEGA8, np.array(bits))
    re, ce, Qe = _exact_refit(S, OMEGA8, bits, G8)
    for i in range(8):
        assert abs(r[i] - float(re[i])) <= 1e-14 * float(re[i])
        if bits[i] == 16:
            assert np.all(Q[i] == 0)
            assert np.array_equal(piv[i], S[i].astype(np.float16))
        else:
            assert [int(x) for x in Q[i]] == Qe[i]
    for j in range(8):
        assert abs(c[j] - float(ce[j])) <= 1e-13 * float(ce[j])


def test_plain_update_identity_and_delta_property():
    rng = np.random.default_rng(3)
    S = rng.standard_normal((5, D, D))
    k = rng.standard_normal((5, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((5, D))
    ones = np.ones((5, D))
    # beta = 0 and D = I: the state is unchanged
    assert np.array_equal(P.gated_delta_update(S, k, v, ones, np.zeros(5)), S)
    # unit k and beta = 1: k^T S_t = v^T (the association is written exactly)
    St = P.gated_delta_update(S, k, v, ones, np.ones(5))
    assert np.abs(np.einsum("bi,bij->bj", k, St) - v).max() <= 1e-12
    # the decay acts on key rows: a zero key row of D leaves beta k v^T - beta k k^T D S
    dec = np.ones((5, D))
    dec[:, 7] = 0.0
    St = P.gated_delta_update(S, k, v, dec, np.zeros(5))
    assert np.all(St[:, 7] == 0) and np.array_equal(St[:, 8], S[:, 8])


def test_plain_restore_hand_example():
    bits = np.array([6, 16, 2, 4])
    u = np.zeros((4, 4), np.int64)
    u[0] = [32, 33, 31, 63]          # Q = 0, 1, -1, 31
    u[2] = [1, 2, 3, 2]              # Q = -1, 0, 1, 0
    u[3] = [8, 15, 1, 9]             # Q = 0, 7, -7, 1
    r = np.array([0.5, 0.0, 2.0, 0.25])
    c = np.array([1.0, 2.0, 4.0, 8.0])
    piv = np.zeros((4, 4), np.float16)
    piv[1] = [1.5, -2.0, 0.25, 3.0]
    X = P.restore(u, r, c, piv, bits)
    assert np.array_equal(X, [[0, 1, -2, 124], [1.5, -2, 0.25, 3], [-2, 0, 8, 0], [0, 3.5, -7, 2]])


def test_plain_least_squares_step_is_weighted_optimum():
    rng = np.random.default_rng(9)
    S = rng.standard_normal((2, D, D)) * rng.lognormal(0, 1, (2, 1, D))
    omega = rng.lognormal(0, 1, (2, D))
    bits = np.full((2, D), 6)
    Q0, r, c0, _ = P.refit(S, omega, bits, n_ls=0)
    _, _, c1, _ = P.refit(S, omega, bits, n_ls=1)
    for h in range(2):
        for j in range(0, D, 17):
            a = (np.sqrt(omega[h]) * r[h] * Q0[h, :, j])[:, None]
            b = np.sqrt(omega[h]) * S[h, :, j]
            assert abs(np.linalg.lstsq(a, b, rcond=None)[0][0] - c1[h, j]) <= 1e-12 * abs(c1[h, j])


def distance(widx, t=0):
    """Both oracles' decode step from one packed state of workload `widx` (request 0,
    256 FP32 warm-up steps, quantised by the float32 oracle): relative distances of r,
    c, the readout and the dequantised states, and the fraction of codes that differ."""
    w = W.WORKLOADS[widx]
    rb, om = W.row_bits(w), W.omega(w)
    S0 = T.warm_state(widx, (0,))
    u, r, c, piv = O.refit(S0, om, rb)
    x = T.inputs_for(w, "decode", t, [0])
    dec = O.gate_rows(x.gate, w.kind, D)
    u32, r32, c32, p32, o32, _ = O.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v, dec, x.beta)
    Q64, r64, c64, p64, o64, _ = P.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v, dec, x.beta)
    quant = rb != 16
    u64 = P.biased_codes(Q64, rb)
    nq = int(np.broadcast_to(quant[..., None], u32.shape).sum())
    diff = (u32 != u64) & quant[..., None]
    S32 = O.dequantize(u32, r32, c32, p32, rb).astype(np.float64)
    S64 = P.dequantised(Q64, r64, c64, p64, rb)
    rq = np.broadcast_to(quant, r32.shape)
    return {
        "r_rel_max": float(np.max(np.abs(r32[rq] - r64[rq]) / np.abs(r64[rq]))),
        "c_rel_max": float(np.max(np.abs(c32 - c64) / np.maximum(np.abs(c64), 1e-300))),
        "o_rel_l2": T.rel_l2(o32, o64),
        "state_rel_l2": T.rel_l2(S32, S64),
        "code_diff_frac": int(diff.sum()) / nq,
        "code_diff_max": int(np.abs(u32 - u64)[diff].max()) if diff.any() else 0,
    }


@pytest.mark.parametrize("widx", [1, 2])
def test_float32_order_against_plain_rule(widx):
    d = distance(widx)
    print(f"\nfloat32 oracle vs plain float64 rule, {W.WORKLOADS[widx].name}, one step: "
          + ", ".join(f"{k} {v:.3g}" for k, v in d.items()))
    assert d["r_rel_max"] <= 1e-6
    assert d["o_rel_l2"] <= 1e-6
    assert d["code_diff_max"] <= 1
    assert d["state_rel_l2"] <= 1e-4
