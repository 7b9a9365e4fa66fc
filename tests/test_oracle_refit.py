"""Pins of the oracle's dual-axis refit (row scale, column scale start, two weighted
least-squares steps, final codes) against exact rational arithmetic, closed forms and
the properties the rule guarantees (bloombook section 4; singularity-lens dual-axis
paragraph)."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import stq_oracle as O

F32 = np.float32

# omega with omega_i / mean = s_i^2 for rational s_i, so g_i = 1/s_i is exact
OMEGA8 = np.array([0.25, 1.0, 0.25, 4.0, 1.0, 0.25, 1.0, 0.25], F32)
G8 = [Fraction(2), Fraction(1), Fraction(2), Fraction(1, 2), Fraction(1), Fraction(2), Fraction(1), Fraction(2)]


def test_row_gain_closed_form():
    g = O.row_gain(OMEGA8)
    assert [Fraction(float(x)) for x in g] == G8
    assert np.all(O.row_gain(np.full((3, 128), 7.5, F32)) == 1)


def _exact_refit(S, omega, bits, g):
    """The refit rule in exact rational arithmetic (no rounding except the integer
    code decision, half to even)."""
    d = len(S)
    S = [[Fraction(float(x)) for x in row] for row in S]
    qm = [0 if b == 16 else 2 ** (b - 1) - 1 for b in bits]
    piv = [b == 16 for b in bits]
    r = [Fraction(0) if piv[i] else sum(abs(x) for x in S[i]) / d * g[i] for i in range(d)]
    y = [[(S[i][j] / r[i]) if r[i] != 0 else Fraction(0) for j in range(d)] for i in range(d)]
    c = [max([abs(y[i][j]) / qm[i] for i in range(d) if not piv[i]] + [Fraction(0)]) for j in range(d)]
    w = [Fraction(float(omega[i])) * r[i] * r[i] for i in range(d)]

    def quant(c):
        Q = [[0] * d for _ in range(d)]
        for j in range(d):
            for i in range(d):
                if piv[i] or c[j] == 0:
                    continue
                Q[i][j] = max(-qm[i], min(qm[i], round(y[i][j] / c[j])))
        return Q

    for _ in range(2):
        Q = quant(c)
        for j in range(d):
            num = sum(w[i] * Q[i][j] * y[i][j] for i in range(d))
            den = sum(w[i] * Q[i][j] * Q[i][j] for i in range(d))
            if den > 0:
                c[j] = num / den
    return r, c, quant(c)


@pytest.mark.parametrize("seed,bits", [
    (0, [8] * 8), (1, [6] * 8), (2, [4] * 8), (3, [2] * 8),
    (4, [2, 4, 6, 8, 16, 8, 6, 4]), (5, [6, 16, 6, 6, 4, 8, 16, 2]),
])
def test_refit_matches_exact_rational_rule(seed, bits):
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal((8, 8)) * rng.lognormal(0, 1, (8, 1)) * rng.lognormal(0, 1, (1, 8))).astype(F32)
    u, r, c, piv = O.refit(S, OMEGA8, np.array(bits))
    re, ce, Qe = _exact_refit(S, OMEGA8, bits, G8)
    for i in range(8):
        assert abs(float(r[i]) - float(re[i])) <= 4e-7 * float(re[i])
    for j in range(8):
        assert abs(float(c[j]) - float(ce[j])) <= 1e-5 * float(ce[j])
    bias = O.bias_of(np.array(bits))
    for i in range(8):
        if bits[i] == 16:
            assert np.all(u[i] == 0)
            assert np.array_equal(piv[i], S[i].astype(np.float16))
        else:
            assert list(u[i] - bias[i]) == Qe[i]


def test_half_step_bound_and_no_clip_at_start():
    rng = np.random.default_rng(7)
    S = (rng.standard_normal((16, 128, 128)) * rng.lognormal(0, 1, (16, 128, 1))).astype(F32)
    omega = rng.lognormal(0, 1, (16, 128)).astype(F32)
    bits = np.array([[[2, 4, 6, 8][h % 4]] * 128 for h in range(16)])
    for n_ls in (0, 2):
        u, r, c, _ = O.refit(S, omega, bits, n_ls=n_ls)
        Q = u - O.bias_of(bits)[..., None]
        qm = O.qmax_of(bits)[..., None]
        rec = r[..., :, None].astype(np.float64) * c[..., None, :] * Q
        step = r[..., :, None].astype(np.float64) * c[..., None, :]
        inside = np.abs(Q) < qm
        err = np.abs(S - rec)
        assert np.all(err[inside] <= 0.5 * step[inside] * (1 + 1e-5))
        if n_ls == 0:
            # start scale from the column maximum: nothing clips, and every column's
            # largest code reaches qmax
            x = S / step
            assert np.all(np.abs(x) <= qm * (1 + 1e-5) + 1e-6)
            assert np.all(np.max(np.abs(Q), axis=-2) == qm[:, 0])


def test_least_squares_step_is_weighted_optimum():
    # c after one step minimises sum_i omega_i (S_ij - r_i c Q_ij)^2 for the codes of the
    # previous scale; checked column by column against numpy's lstsq
    rng = np.random.default_rng(8)
    S = (rng.standard_normal((4, 128, 128)) * rng.lognormal(0, 1, (4, 1, 128))).astype(F32)
    omega = rng.lognormal(0, 1, (4, 128)).astype(F32)
    bits = np.full((4, 128), 6)
    u0, r, c0, _ = O.refit(S, omega, bits, n_ls=0)
    _, _, c1, _ = O.refit(S, omega, bits, n_ls=1)
    Q0 = (u0 - 32).astype(np.float64)
    for h in range(4):
        sw = np.sqrt(omega[h].astype(np.float64))
        for j in range(0, 128, 7):
            a = (sw * r[h].astype(np.float64) * Q0[h, :, j])[:, None]
            b = sw * S[h, :, j].astype(np.float64)
            sol = np.linalg.lstsq(a, b, rcond=None)[0][0]
            assert abs(c1[h, j] - sol) <= 2e-5 * abs(sol)


def test_scaling_and_sign_symmetry_exact():
    rng = np.random.default_rng(9)
    S = rng.standard_normal((3, 128, 128)).astype(F32)
    omega = rng.lognormal(0, 1, (3, 128)).astype(F32)
    bits = np.array([[6] * 128, [4] * 128, [2, 8] * 64])
    u, r, c, _ = O.refit(S, omega, bits)
    u2, r2, c2, _ = O.refit(S * F32(8), omega, bits)
    assert np.array_equal(u, u2) and np.array_equal(r * F32(8), r2) and np.array_equal(c, c2)
    u3, r3, c3, _ = O.refit(-S, omega, bits)
    bias = O.bias_of(bits)[..., None]
    assert np.array_equal(u3 - bias, -(u - bias)) and np.array_equal(r3, r) and np.array_equal(c3, c)


def test_rank_one_outer_product_is_reconstructed():
    # S_ij = s_i t_j with |s_i| constant and equal omega: every code sits at +-qmax and
    # the dequantised state equals S up to float32 rounding
    rng = np.random.default_rng(10)
    s = np.where(rng.random(128) < 0.5, -1.5, 1.5)
    t = rng.standard_normal(128)
    S = np.outer(s, t).astype(F32)
    bits = np.full(128, 6)
    u, r, c, piv = O.refit(S, np.ones(128, F32), bits)
    assert np.all(np.abs(u - 32) == 31)
    back = O.dequantize(u, r, c, piv, bits)
    assert np.max(np.abs(back - S)) <= 1e-6 * np.max(np.abs(S))


def test_zero_state_and_zero_rows():
    bits = np.full(128, 4)
    u, r, c, _ = O.refit(np.zeros((128, 128), F32), np.ones(128, F32), bits)
    assert np.all(u == 8) and np.all(r == 0) and np.all(c == 0)
    S = np.random.default_rng(11).standard_normal((128, 128)).astype(F32)
    S[5] = 0
    S[:, 9] = 0
    u, r, c, _ = O.refit(S, np.ones(128, F32), bits)
    assert r[5] == 0 and np.all(u[5] == 8) and c[9] == 0 and np.all(u[:, 9] == 8)
    assert np.all(O.dequantize(u, r, c, np.zeros((128, 128), np.float16), bits)[5] == 0)


def test_subnormal_scale_counts_as_zero():
    # a column of subnormal values: its start scale is below 2^-126, so its codes are 0
    # rather than the NaN that 0 * (1/c) = 0 * inf would give
    S = np.random.default_rng(12).standard_normal((128, 128)).astype(F32)
    S[:, 3] = np.float32(1e-44)
    u, r, c, _ = O.refit(S, np.ones(128, F32), np.full(128, 6))
    assert np.all(np.isfinite(c)) and np.all(u[:, 3] == 32) and np.all((u >= 1) & (u <= 63))


def test_dequantize_hand_example():
    # X_ij = r_i c_j z_ij (bloombook section 4) with z = u - 2^(b-1)
    bits = np.array([4, 4, 16, 2])
    u = np.array([[8, 9, 7, 15], [1, 8, 8, 8], [0, 0, 0, 0], [1, 2, 3, 2]])
    r = np.array([0.5, 2.0, 0.0, 1.0], F32)
    c = np.array([1.0, 0.25, 4.0, 2.0], F32)
    piv = np.zeros((4, 4), np.float16)
    piv[2] = [1.5, -2.0, 0.0, 65504.0]
    S = O.dequantize(u, r, c, piv, bits)
    expect = np.array([[0, 0.125, -2, 7], [-14, 0, 0, 0], [1.5, -2.0, 0.0, 65504.0], [-1, 0, 4, 0]], F32)
    assert np.array_equal(S, expect)
    S2 = O.dequantize(u, r, c, piv, bits, decay=np.array([0.5, 0.5, 0.5, 2.0], F32))
    assert np.array_equal(S2, expect * np.array([0.5, 0.5, 0.5, 2.0], F32)[:, None])


# ---------------------------------------------------------------------------------
# scalar twin: the same rule with Python loops over float32 scalars on tiny heads,
# to catch axis and broadcasting slips in the vectorised oracle
# ---------------------------------------------------------------------------------

def rn32(x: Fraction) -> np.float32:
    """Exact rational -> nearest float32, ties to even (normal and subnormal range)."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    if Fraction(2) ** e > x:
        e -= 1
    e = max(e, -126)                       # subnormals share the 2^-149 step
    scaled = x / Fraction(2) ** (e - 23)   # in [2^23, 2^24) for normal numbers
    m = scaled.numerator // scaled.denominator
    rem = scaled - m
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and m % 2 == 1):
        m += 1
    return np.float32(sign * float(Fraction(m) * Fraction(2) ** (e - 23)))


def fma_exact(a, b, c):
    return rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _tsum(xs):
    xs = list(xs)
    while len(xs) > 1:
        xs = [xs[2 * i] + xs[2 * i + 1] for i in range(len(xs) // 2)]
    return xs[0]


def _tdot(a, b):
    a, b = list(a), list(b)
    return _tsum([fma_exact(a[2 * m], b[2 * m], a[2 * m + 1] * b[2 * m + 1]) for m in range(len(a) // 2)])


def _scalar_refit(S, omega, bits):
    d = len(S)
    f = np.float32
    w64 = [float(x) for x in omega]
    acc = 0.0
    for x in w64:
        acc += x
    mean = acc / d
    g = [f(1.0 / np.sqrt(x / mean)) for x in w64]
    piv = [b == 16 for b in bits]
    qm = [0 if p else 2 ** (b - 1) - 1 for b, p in zip(bits, piv)]
    r, inv_r = [], []
    for i in range(d):
        m = _tsum([abs(S[i][j]) for j in range(d)]) * f(1.0 / d)
        ri = f(0) if piv[i] else m * g[i]
        r.append(ri)
        inv_r.append(f(1) / ri if ri >= f(2.0 ** -126) else f(0))
    y = [[S[i][j] * inv_r[i] for j in range(d)] for i in range(d)]
    c = []
    for j in range(d):
        best = f(0)
        for i in range(d):
            if not piv[i]:
                best = max(best, abs(y[i][j]) * (f(1) / f(qm[i])))
        c.append(best)
    b = [omega[i] * (r[i] * r[i]) for i in range(d)]

    def quant(c):
        Q = [[f(0)] * d for _ in range(d)]
        for j in range(d):
            ic = f(1) / c[j] if c[j] >= f(2.0 ** -126) else f(0)
            for i in range(d):
                x = float(y[i][j]) * float(ic)
                Q[i][j] = f(max(-qm[i], min(qm[i], np.rint(x))))
        return Q

    for _ in range(2):
        Q = quant(c)
        for j in range(d):
            p = [b[i] * Q[i][j] for i in range(d)]
            num = _tdot(p, [y[i][j] for i in range(d)])
            den = _tdot(p, [Q[i][j] for i in range(d)])
            if den > 0:
                c[j] = num / den
    return r, c, quant(c)


@pytest.mark.parametrize("seed", range(6))
def test_vectorised_refit_equals_scalar_twin(seed):
    rng = np.random.default_rng(100 + seed)
    d = 8
    S = (rng.standard_normal((d, d)) * rng.lognormal(0, 1, (d, 1))).astype(F32)
    omega = rng.lognormal(0, 1, d).astype(F32)
    bits = list(rng.choice([2, 4, 6, 8, 16], d))
    u, r, c, _ = O.refit(S, omega, np.array(bits))
    rs, cs, Qs = _scalar_refit([[F32(x) for x in row] for row in S], [F32(x) for x in omega], bits)
    assert [F32(x) for x in r] == rs
    assert [F32(x) for x in c] == cs
    bias = O.bias_of(np.array(bits))
    for i in range(d):
        if bits[i] != 16:
            assert [int(x) for x in u[i] - bias[i]] == [int(x) for x in Qs[i]]


def test_fma32_is_correctly_rounded():
    # against exact rational arithmetic, on random operands and on products that land
    # on or next to float32 rounding midpoints
    rng = np.random.default_rng(13)
    a = rng.standard_normal(3000).astype(F32)
    b = (rng.standard_normal(3000) * np.exp2(rng.integers(-30, 30, 3000))).astype(F32)
    c = rng.standard_normal(3000).astype(F32)
    # c = -RN(a*b) + tiny makes the result depend on the low product bits
    c[:1000] = (-(a[:1000] * b[:1000])).astype(F32)
    c[1000:1500] = (a[1000:1500] * b[1000:1500] * F32(3)).astype(F32)
    # midpoint cases: a*b exactly halfway between floats of c's binade
    c[1500:1600] = F32(1.0)
    a[1500:1600] = F32(2.0 ** -24)
    b[1500:1600] = np.where(rng.random(100) < 0.5, 1.0, -1.0).astype(F32) * F32(1 + 2.0 ** -23)
    got = O.fma32(a, b, c)
    for i in range(3000):
        assert got[i] == fma_exact(a[i], b[i], c[i]), i


def test_tree_dot_pairs_products_by_fma():
    rng = np.random.default_rng(14)
    a = rng.standard_normal((5, 16)).astype(F32)
    b = rng.standard_normal((5, 16)).astype(F32)
    got = O.tree_dot(a, b, axis=1)
    for r in range(5):
        assert got[r] == _tdot(a[r], b[r])
    assert np.allclose(got, (a.astype(np.float64) * b).sum(1), atol=1e-5)
