"""Pins of the oracle's whole decode step: the order the pages give (restore, update
in floating point, read out, requantise: singularity-lens decode-order paragraph) and
the error recurrence E_t = A_t E_{t-1} + eps_t (bloombook section 2)."""
import numpy as np

from oracle import stq_oracle as O

F32 = np.float32


def _inputs(rng, n, d, kind):
    q = rng.standard_normal((n, d)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((n, d)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((n, d))
    beta = 1 / (1 + np.exp(-rng.standard_normal(n)))
    if kind == "gdn":
        dec = np.repeat(np.exp(rng.uniform(-0.2, -0.001, n))[:, None], d, 1)
    else:
        dec = np.exp(rng.uniform(-0.5, -0.0005, (n, d)))
    return [a.astype(F32) for a in (q, k, v, dec, beta)]


def _run_pair(kind, bits, steps=64, n=4, d=128, seed=0):
    rng = np.random.default_rng(seed)
    omega = rng.lognormal(0, 1, (n, d)).astype(F32)
    S0 = np.zeros((n, d, d), F32)
    for _ in range(64):
        q, k, v, dec, beta = _inputs(rng, n, d, kind)
        S0, _ = O.fp32_step(S0, q, k, v, dec, beta)
    u, r, c, piv = O.refit(S0, omega, bits)
    Sf = O.dequantize(u, r, c, piv, bits)   # both paths start from the same state
    hist = []
    for _ in range(steps):
        q, k, v, dec, beta = _inputs(rng, n, d, kind)
        Shat_prev = O.dequantize(u, r, c, piv, bits)
        u, r, c, piv, o, X = O.decode_step(u, r, c, piv, bits, omega, q, k, v, dec, beta)
        Shat = O.dequantize(u, r, c, piv, bits)
        Sf_prev = Sf
        Sf, of = O.fp32_step(Sf, q, k, v, dec, beta)
        hist.append(dict(q=q, k=k, dec=dec, beta=beta, X=X, Shat=Shat, Shat_prev=Shat_prev,
                         Sf=Sf, Sf_prev=Sf_prev, o=o, of=of))
    return hist


def test_error_recurrence_on_paired_runs():
    bits = np.full((4, 128), 6)
    for t, h in enumerate(_run_pair("gdn", bits)):
        n, d = h["Sf"].shape[:2]
        for m in range(n):
            kk = h["k"][m].astype(np.float64)
            A = (np.eye(d) - float(h["beta"][m]) * np.outer(kk, kk)) @ np.diag(h["dec"][m].astype(np.float64))
            E = h["Shat"][m].astype(np.float64) - h["Sf"][m]
            Ep = h["Shat_prev"][m].astype(np.float64) - h["Sf_prev"][m]
            eps = h["Shat"][m].astype(np.float64) - h["X"][m]
            resid = np.linalg.norm(E - A @ Ep - eps)
            assert resid <= 1e-5 * np.linalg.norm(h["Sf"][m]), (t, m, resid)


def test_readout_uses_updated_state_before_requantisation():
    bits = np.full((4, 128), 4)
    for h in _run_pair("kda", bits, steps=8):
        for m in range(4):
            pre = h["X"][m].astype(np.float64).T @ h["q"][m]
            post = h["Shat"][m].astype(np.float64).T @ h["q"][m]
            assert np.max(np.abs(h["o"][m] - pre)) <= 1e-5 * np.max(np.abs(pre))
            assert np.max(np.abs(post - pre)) > 100 * np.max(np.abs(h["o"][m] - pre))


def test_all_pivot_state_tracks_fp32():
    bits = np.full((4, 128), 16)
    hist = _run_pair("kda", bits, steps=64)
    last = hist[-1]
    rel = np.linalg.norm(last["Shat"] - last["Sf"]) / np.linalg.norm(last["Sf"])
    assert rel <= 1e-3, rel
    assert np.all(last["Shat"] == last["Shat"].astype(np.float16).astype(F32))


def test_quantised_state_stays_close_at_8_bits():
    # sanity of the whole loop: 8-bit codes with the refit keep the chain near FP32
    bits = np.full((4, 128), 8)
    hist = _run_pair("gdn", bits, steps=32)
    last = hist[-1]
    rel = np.linalg.norm(last["Shat"] - last["Sf"]) / np.linalg.norm(last["Sf"])
    assert rel < 0.05, rel


# ---------------------------------------------------------------------------------
# scalar twin of the whole step: Python loops over float32 scalars on 4x4 and 8x8
# heads (restore with the decay folded into r, delta rule with fused pairs, readout,
# requantisation), to catch a transposed operand, a wrong axis or a dropped term in
# the vectorised oracle
# ---------------------------------------------------------------------------------
import math  # noqa: E402

import pytest  # noqa: E402

from test_oracle_refit import _scalar_refit, _tdot, fma_exact  # noqa: E402


def _scalar_absmax(S, bits):
    f = np.float32
    d = len(S)
    r, Q = [], []
    for i in range(d):
        if bits[i] == 16:
            r.append(f(0))
            Q.append([f(0)] * d)
            continue
        qm = 2 ** (bits[i] - 1) - 1
        ri = max(abs(S[i][j]) for j in range(d)) * (f(1) / f(qm))
        ir = f(1) / ri if ri >= f(2.0 ** -126) else f(0)
        r.append(ri)
        Q.append([f(max(-qm, min(qm, np.rint(float(S[i][j]) * float(ir))))) for j in range(d)])
    c = [f(1) if any(b != 16 for b in bits) else f(0)] * d
    return r, c, Q


def _scalar_step(u, r, c, piv, bits, omega, q, k, v, dec, beta, scheme):
    f = np.float32
    d = len(bits)
    Sp = [[f(0)] * d for _ in range(d)]
    for i in range(d):
        for j in range(d):
            if bits[i] == 16:
                Sp[i][j] = dec[i] * f(piv[i][j])
            else:
                Qij = f(int(u[i][j]) - 2 ** (bits[i] - 1))
                Sp[i][j] = (Qij * (dec[i] * r[i])) * c[j]
    # u_j = sum_i k_i S'_ij, delta_j = beta (v_j - u_j), S_ij = S'_ij + k_i delta_j
    uu = [_tdot(k, [Sp[i][j] for i in range(d)]) for j in range(d)]
    delta = [beta * (v[j] - uu[j]) for j in range(d)]
    S = [[fma_exact(k[i], delta[j], Sp[i][j]) for j in range(d)] for i in range(d)]
    # o_j = sum_i q_i S_ij: exact products, one rounding to float64, then to float32
    o = [f(math.fsum(float(q[i]) * float(S[i][j]) for i in range(d))) for j in range(d)]
    if scheme == "row_absmax":
        r2, c2, Q2 = _scalar_absmax(S, bits)
    else:
        r2, c2, Q2 = _scalar_refit(S, omega, bits)
    piv2 = [[np.float16(S[i][j]) if bits[i] == 16 else np.float16(0) for j in range(d)] for i in range(d)]
    return S, o, r2, c2, Q2, piv2


@pytest.mark.parametrize("scheme", ["stepquant", "row_absmax"])
@pytest.mark.parametrize("d,seed", [(4, 0), (4, 1), (4, 2), (8, 3), (8, 4), (8, 5)])
def test_decode_step_equals_scalar_twin(scheme, d, seed):
    rng = np.random.default_rng(700 + seed)
    S0 = (rng.standard_normal((d, d)) * rng.lognormal(0, 1, (d, 1))).astype(F32)
    omega = rng.lognormal(0, 1, d).astype(F32)
    bits = np.array(rng.choice([2, 4, 6, 8, 16], d))
    bits[0] = 6                                   # at least one quantised row
    quant = (lambda S: O.absmax_quantise(S, bits)) if scheme == "row_absmax" else (lambda S: O.refit(S, omega, bits))
    u, r, c, piv = quant(S0)
    q = rng.standard_normal(d).astype(F32)
    k = rng.standard_normal(d); k = (k / np.linalg.norm(k)).astype(F32)
    v = rng.standard_normal(d).astype(F32)
    dec = np.exp(rng.uniform(-0.5, -0.01, d)).astype(F32)      # per key row (KDA form)
    beta = F32(rng.uniform(0.1, 0.9))
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, bits, omega, q, k, v, dec, beta, scheme=scheme)
    Ss, os_, rs, cs, Qs, ps = _scalar_step(u, r, c, piv, list(bits), [F32(x) for x in omega],
                                          q, k, v, dec, beta, scheme)
    assert [[F32(x) for x in row] for row in X] == Ss
    assert [F32(x) for x in o] == os_
    assert [F32(x) for x in r2] == rs
    assert [F32(x) for x in c2] == cs
    bias = O.bias_of(bits)
    for i in range(d):
        if bits[i] != 16:
            assert [int(x) for x in u2[i] - bias[i]] == [int(x) for x in Qs[i]]
        else:
            assert [np.float16(x) for x in p2[i]] == ps[i]
