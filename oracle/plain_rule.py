"""The decode step's rule in its literal form, in float64 (test infrastructure only).

`stq_oracle` fixes one float32 evaluation order for the step (balanced tree sums with
fused product pairs, the decay folded into the row scale, the least-squares sums taken
from r_i * y_ij), because packed codes are compared bit for bit and a one-ulp change
in a column sum moves codes far from any rounding boundary. That order is a reading:
the pages fix none. This module evaluates the same rule as plainly as it is written,
so the tests can measure how far the shipped float32 arithmetic sits from it:

  * every quantity is float64; sums are plain numpy sums (no tree, no fused pairs);
  * the restore is X_ij = r_i c_j z_ij (bloombook.cn tutorial, section 4: dual-axis
    scales), then the decay acts as the matrix D_t on the restored state;
  * the update is the printed matrix form S_t = (I - beta k k^T) D_t S_{t-1}
    + beta k v^T (bloombook section 2), the readout o = S_t^T q from the updated state
    before requantisation (singularity-lens.com summary, decode-order paragraph);
  * the refit is the build's rule with S itself in every sum: r_i = mean_j |S_ij| g_i,
    g_i = (omega_i / mean omega)^(-1/2); c_j starts at max_i |S_ij| / (r_i qmax_i) over
    the quantised rows; then twice c_j = sum_i omega_i r_i Q_ij S_ij /
    sum_i omega_i r_i^2 Q_ij^2 with Q_ij = clamp(rint(S_ij / (r_i c_j)), -qmax_i,
    qmax_i) (bloombook section 4; singularity-lens dual-axis paragraph); the stored
    codes are requantised with the final c. FP16 pivot rows (ai-trend.me review,
    Method) are rounded to binary16 and take no part in the refit.

Degenerate cases follow `stq_oracle`: a zero row scale gives a zero row of codes, a
zero column scale a zero column, a zero least-squares denominator keeps the column
scale. The scales stay float64 (they are not rounded to the pool's storage type).

Nothing here is imported by the library, and nothing here imports it.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
PIVOT_BITS = 16


def _qmax(row_bits):
    b = np.asarray(row_bits, dtype=np.int64)
    return np.where(b == PIVOT_BITS, 0, (1 << (b - 1)) - 1).astype(F64)


def _bias(row_bits):
    b = np.asarray(row_bits, dtype=np.int64)
    return np.where(b == PIVOT_BITS, 0, 1 << (b - 1))


def restore(u, r, c, piv, row_bits):
    """X_ij = r_i c_j z_ij for quantised rows (z = u - 2^(b-1)); pivot rows are their
    binary16 values. u [..., d, d] biased codes, r/c [..., d], piv [..., d, d]."""
    row_bits = np.asarray(row_bits)
    pivot = (row_bits == PIVOT_BITS)[..., None]
    z = (np.asarray(u, dtype=np.int64) - _bias(row_bits)[..., None]).astype(F64)
    X = np.asarray(r, F64)[..., :, None] * np.asarray(c, F64)[..., None, :] * z
    return np.where(pivot, np.asarray(piv).astype(F64), X)


def gated_delta_update(S_prev, k, v, decay, beta):
    """S_t = (I - beta k k^T) D_t S_{t-1} + beta k v^T with D_t = diag(decay), as
    matrices in float64. S_prev [..., d, d]; k, v, decay [..., d]; beta [...]."""
    S_prev = np.asarray(S_prev, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    beta = np.asarray(beta, F64)[..., None, None]
    d = S_prev.shape[-1]
    A = np.eye(d) - beta * (k[..., :, None] * k[..., None, :])
    DS = np.asarray(decay, F64)[..., :, None] * S_prev
    return A @ DS + beta * (k[..., :, None] * v[..., None, :])


def readout(S, q):
    """o_j = sum_i q_i S_ij."""
    return np.einsum("...ij,...i->...j", np.asarray(S, F64), np.asarray(q, F64))


def _quantise(S, r, c, qm):
    """Q_ij = clamp(rint(S_ij / (r_i c_j)), -qmax_i, qmax_i); 0 where r_i c_j = 0."""
    rc = r[..., :, None] * c[..., None, :]
    safe = np.where(rc > 0, rc, 1.0)
    x = np.where(rc > 0, S / safe, 0.0)
    return np.clip(np.rint(x), -qm[..., :, None], qm[..., :, None])


def refit(S, omega, row_bits, n_ls=2):
    """The dual-axis refit of a float64 state, every sum a plain float64 sum.

    Returns (Q [..., d, d] float64 integers, r [..., d], c [..., d],
    piv [..., d, d] binary16)."""
    S = np.asarray(S, F64)
    row_bits = np.asarray(row_bits)
    pivot = row_bits == PIVOT_BITS
    qm = _qmax(row_bits)
    om = np.asarray(omega, F64)
    g = 1.0 / np.sqrt(om / om.mean(axis=-1, keepdims=True))
    r = np.where(pivot, 0.0, np.abs(S).mean(axis=-1) * g)
    # column start: the largest |S_ij| / (r_i qmax_i) over the quantised rows
    den0 = r * qm
    ok = (den0 > 0)[..., :, None]
    ratio = np.where(ok, np.abs(S) / np.where(ok, den0[..., :, None], 1.0), 0.0)
    c = ratio.max(axis=-2)
    wr = om * r                     # omega_i r_i
    for _ in range(n_ls):
        Q = _quantise(S, r, c, qm)
        num = np.sum(wr[..., :, None] * Q * S, axis=-2)
        den = np.sum((wr * r)[..., :, None] * Q * Q, axis=-2)
        c = np.where(den > 0, num / np.where(den > 0, den, 1.0), c)
    Q = _quantise(S, r, c, qm)
    Q = np.where(pivot[..., None], 0.0, Q)
    piv = np.where(pivot[..., None], S, 0.0).astype(np.float16)
    return Q, r, c, piv


def decode_step(u, r, c, piv, row_bits, omega, q, k, v, decay, beta, n_ls=2):
    """One decode step of the literal rule from a packed state (u, r, c, piv):
    restore, gated delta update, readout, refit. decay is per key row [..., d].

    Returns (Q, r, c, piv, o, S) with S the updated float64 state before
    requantisation."""
    X = restore(u, r, c, piv, row_bits)
    S = gated_delta_update(X, k, v, decay, beta)
    o = readout(S, q)
    Q2, r2, c2, piv2 = refit(S, omega, row_bits, n_ls=n_ls)
    return Q2, r2, c2, piv2, o, S


def biased_codes(Q, row_bits):
    """Stored codes u = Q + 2^(b-1) (0 on pivot rows)."""
    row_bits = np.asarray(row_bits)
    u = Q.astype(np.int64) + _bias(row_bits)[..., None]
    return np.where((row_bits == PIVOT_BITS)[..., None], 0, u)


def dequantised(Q, r, c, piv, row_bits):
    """The state the stored triple stands for, in float64."""
    return restore(biased_codes(Q, row_bits), r, c, piv, row_bits)
