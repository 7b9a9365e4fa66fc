"""Oracle of the offline, lifetime-aware bit allocation (test infrastructure only; see
the package docstring).

The pages' offline stage (bloombook section 3 and section 4, "time" half;
singularity-lens calibration paragraph; ai-trend review, Method (1)):
  * every unit u (a head for GDN, a key row for KDA) gets a lifetime weight
    L_u = sum_{j<J} exp(2 j l_u), l_u its mean log-retention over the calibration data,
    J a finite horizon;
  * each candidate width b gives a distortion D_u(b) of the unit's calibration states
    quantised at b: a row-sensitivity (omega) weighted mean squared error for GDN heads,
    a plain per-row mean squared error for KDA rows;
  * widths minimise sum_u L_u D_u(b_u) under a mean-bit budget, candidates {2,4,6,8}
    for a 4-bit budget and {4,6,8} for a 6-bit one;
  * a few highest-risk units are kept in FP16 as pivots.

Readings where the pages are silent:
  * J = 1024, the decode length of the pages' throughput protocol.
  * Risk of a unit = L_u D_u(b_max): the weighted distortion it keeps even at the widest
    integer width (the pages keep in FP16 the units that a few more bits would not rescue).
    The n_pivots riskiest units (ties: lower unit index first) become pivots first.
  * The remaining units share the budget: sum of their widths <= budget * (their count),
    solved exactly by dynamic programming over the total width in steps of 2 bits;
    among equal costs the narrower width and then the smaller total win.
  * D_u(b) is measured with the method's own quantiser (the dual-axis refit) on states
    whose every unit has width b.
  * Distortions and costs are float64; row errors are float32 tree sums of the squared
    float32 differences (the same tree as every other row sum of the oracle).
"""
import math

import numpy as np

from .stq_oracle import tree_sum

F32 = np.float32
F64 = np.float64
PIVOT_BITS = 16


def lifetime_weight(ell, horizon=1024):
    """L_u = sum_{j=0}^{J-1} exp(2 j l_u), summed term by term in float64 in the order
    j = 0, 1, ... (bloombook section 3: a geometric series of the squared retention)."""
    ell = np.asarray(ell, dtype=F64)
    j = np.arange(horizon, dtype=F64)
    terms = np.exp(2.0 * j[None, :] * ell.reshape(-1)[:, None])
    return np.cumsum(terms, axis=1)[:, -1].reshape(ell.shape)


def row_sq_error(S, S_hat):
    """e_i = tree sum over the row of (S_ij - S_hat_ij)^2, float32 ([..., d, d] -> [..., d])."""
    d = (np.asarray(S, dtype=F32) - np.asarray(S_hat, dtype=F32)).astype(F32)
    return tree_sum((d * d).astype(F32), axis=-1)


def unit_distortion(kind, row_err, omega):
    """D_u from row errors row_err [N, H, d] (N calibration states):
    GDN head h: sum_n sum_i omega_i e_{n,h,i} / (N d d);  KDA row (h, i):
    sum_n e_{n,h,i} / (N d). Sums are sequential float64 (n outer, i inner).
    Returns [H] (GDN) or [H*d] (KDA) float64."""
    e = np.asarray(row_err, dtype=F64)
    N, H, d = e.shape
    if kind == "gdn":
        w = np.asarray(omega, dtype=F64)                       # [H, d]
        prod = np.transpose(e * w[None], (1, 0, 2)).reshape(H, N * d)   # per head, n outer
        return np.cumsum(prod, axis=1)[:, -1] / float(N * d * d)
    per = np.transpose(e, (1, 2, 0)).reshape(H * d, N)
    return np.cumsum(per, axis=1)[:, -1] / float(N * d)


def allocate(lifetime, dist, cand_bits, budget, n_pivots):
    """Widths per unit: 16 for the n_pivots riskiest units, else a candidate width.
    lifetime [n]; dist [n, n_cand] (D_u(b) per candidate, candidates ascending);
    budget = mean bits over the non-pivot units."""
    L = np.asarray(lifetime, dtype=F64)
    Dm = np.asarray(dist, dtype=F64)
    cand = [int(b) for b in cand_bits]
    assert cand == sorted(cand) and all(b % 2 == 0 for b in cand)
    n = L.shape[0]
    cost = L[:, None] * Dm
    risk = cost[:, -1]
    order = sorted(range(n), key=lambda u: (-risk[u], u))
    pivots = set(order[:n_pivots])
    rest = [u for u in range(n) if u not in pivots]
    m = len(rest)
    K = int(math.floor(budget * m / 2.0))
    ks = [b // 2 for b in cand]
    if ks[0] * m > K:
        raise ValueError("budget below the narrowest candidate width")
    best = np.full(K + 1, np.inf)
    best[0] = 0.0
    choice = np.zeros((m, K + 1), dtype=np.int8)
    for t, u in enumerate(rest):
        new = np.full(K + 1, np.inf)
        ch = np.full(K + 1, -1, dtype=np.int8)
        for ci, k in enumerate(ks):
            v = np.full(K + 1, np.inf)
            v[k:] = best[: K + 1 - k] + cost[u, ci]
            better = v < new
            new[better] = v[better]
            ch[better] = ci
        best = new
        choice[t] = ch
    s = int(np.argmin(best))        # first (smallest total) of the minima
    bits = np.full(n, PIVOT_BITS, dtype=np.int64)
    for t in range(m - 1, -1, -1):
        ci = int(choice[t, s])
        bits[rest[t]] = cand[ci]
        s -= ks[ci]
    return bits


def row_error_at_widths(S, c, omega, cand_bits, scale16=False):
    """Distortion of every row at every candidate width inside a head whose column scales
    are fixed: the head's rows share c_j, so a row's width b only sets how far its codes
    reach (+-qmax_b steps of r_i c_j). For state n, head h, row i and candidate b:
      r_i   = (tree sum_j |S_ij|) * (1/d) * g_i, the refit's row scale (every row, pivot
              rows included: the width they would get is what is measured);
      Q_ij  = clamp(rint((S_ij * fl(1/r_i)) * fl(1/c_j)), -qmax_b, qmax_b) on the exact
              product, 0 when r_i or c_j is below 2^-126;
      e_i(b) = tree sum_j (S_ij - (Q_ij r_i) c_j)^2 in float32, as row_sq_error.
    S [N, H, d, d] float32; c [N, H, d] float32 (the allocated pool's column scales);
    omega [H, d]; scale16: r rounded to binary16 as a compact pool stores it; returns
    [N, H, d, n_cand] float32.
    Reading (the pages name a per-row squared error for KDA units but not the scales it
    is taken under): the allocation is iterated with these in-head errors, since a KDA
    row quantised alone at width b gets a column scale it would not have in a head of
    mixed widths."""
    from .stq_oracle import _recip, row_gain, qmax_of
    S = np.asarray(S, dtype=F32)
    c = np.asarray(c, dtype=F32)
    d = S.shape[-1]
    g = row_gain(omega)
    r = (tree_sum(np.abs(S), axis=-1) * F32(1.0 / d) * g).astype(F32)
    if scale16:
        r = r.astype(np.float16).astype(F32)
    y = (S * _recip(r)[..., :, None]).astype(F32)
    x = y.astype(F64) * _recip(c).astype(F64)[..., None, :]
    out = np.empty(S.shape[:-1] + (len(cand_bits),), F32)
    for ci, b in enumerate(cand_bits):
        qm = float(qmax_of(b))
        Q = np.clip(np.rint(x), -qm, qm).astype(F32)
        S_hat = ((Q * r[..., :, None]).astype(F32) * c[..., None, :]).astype(F32)
        out[..., ci] = row_sq_error(S, S_hat)
    return out
