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
