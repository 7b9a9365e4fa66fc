"""Pins of the oracle's uniform baseline quantiser: symmetric per-key-row absmax INT-b
(singularity-lens calibration and evaluation-setup paragraphs), against the properties
that define an absmax quantiser and against a float64 textbook version of it."""
import numpy as np
import pytest

from oracle import stq_oracle as O

F32 = np.float32


def _state(seed, d=128, n=3):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((n, d, d)).astype(F32)
    S[:, 5, :] *= 10      # an outlier row
    S[:, :, 7] *= 10      # an outlier column
    return S


def _q(u, row_bits):
    return u - O.bias_of(np.asarray(row_bits))[..., None]


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
def test_absmax_maps_row_maximum_to_the_end_of_the_range(bits):
    S = _state(bits)
    rb = np.full((3, 128), bits)
    u, r, c, _ = O.absmax_quantise(S, rb)
    Q = _q(u, rb)
    qm = 2 ** (bits - 1) - 1
    i = np.arange(128)
    jmax = np.argmax(np.abs(S), axis=-1)
    top = np.take_along_axis(Q, jmax[..., None], axis=-1)[..., 0]
    sgn = np.sign(np.take_along_axis(S, jmax[..., None], axis=-1)[..., 0])
    assert np.all(top == sgn * qm)
    assert np.all(np.abs(Q) <= qm)
    assert np.all(c == 1)
    # r_i is the row maximum over qmax to within float32 rounding
    m = np.max(np.abs(S.astype(np.float64)), axis=-1)
    assert np.allclose(r, m / qm, rtol=3e-7, atol=0)
    del i


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
def test_absmax_half_step_bound(bits):
    S = _state(10 + bits)
    rb = np.full((3, 128), bits)
    u, r, c, _ = O.absmax_quantise(S, rb)
    err = np.abs(S.astype(np.float64) - _q(u, rb) * r.astype(np.float64)[..., None])
    assert np.all(err <= 0.5 * r.astype(np.float64)[..., None] * (1 + 1e-6))


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_absmax_agrees_with_float64_textbook_quantiser(bits):
    """np.round(S / (max|S| / qmax)) in float64; the float32 scale and its reciprocal
    may move an element that lies within 1e-5 of a rounding boundary by one."""
    S = _state(20 + bits)
    rb = np.full((3, 128), bits)
    u, _, _, _ = O.absmax_quantise(S, rb)
    qm = 2 ** (bits - 1) - 1
    x = S.astype(np.float64) / (np.max(np.abs(S.astype(np.float64)), axis=-1, keepdims=True) / qm)
    ref = np.round(x)
    diff = _q(u, rb) - ref
    near = np.abs(np.abs(x - np.floor(x)) - 0.5) < 1e-5
    assert np.all((diff == 0) | (near & (np.abs(diff) == 1)))
    assert np.count_nonzero(diff) <= 1e-4 * diff.size


def test_absmax_symmetry_and_power_of_two_scaling():
    S = _state(31)
    rb = np.full((3, 128), 6)
    u, r, _, _ = O.absmax_quantise(S, rb)
    un, rn, _, _ = O.absmax_quantise(-S, rb)
    assert np.array_equal(_q(un, rb), -_q(u, rb)) and np.array_equal(rn, r)
    us, rs, _, _ = O.absmax_quantise(S * F32(8), rb)
    assert np.array_equal(us, u) and np.array_equal(rs, r * F32(8))


def test_absmax_degenerate_rows_and_pivots():
    S = _state(40, n=1)
    S[0, 3, :] = 0
    rb = np.full((1, 128), 4)
    rb[0, 9] = 16
    u, r, c, piv = O.absmax_quantise(S, rb)
    assert r[0, 3] == 0 and np.all(u[0, 3] == 8)           # zero row: Q = 0
    assert r[0, 9] == 0 and np.all(u[0, 9] == 0)           # pivot row: no codes
    assert np.array_equal(piv[0, 9], S[0, 9].astype(np.float16))
    # dequantise with unit column scales is (Q r) exactly
    Sh = O.dequantize(u, r, c, piv, rb)
    mask = rb[0] != 16
    assert np.array_equal(Sh[0][mask], (_q(u, rb)[0] * r[0][:, None]).astype(F32)[mask])


def test_absmax_hand_example():
    """Row (0.5, -1, 0.25, 0) at 8 bits: r = 1 * fl(1/127), codes 64, -127, 32, 0;
    row (3, 1, -2, 0.1) at 4 bits: r = 3 * fl(1/7), codes 7, 2, -5, 0 (worked by hand)."""
    S = np.zeros((1, 4, 4), F32)
    S[0, 0] = [0.5, -1.0, 0.25, 0.0]
    S[0, 2] = [3.0, 1.0, -2.0, 0.1]
    rb = np.array([[8, 6, 4, 4]])
    u, r, _, _ = O.absmax_quantise(S, rb)
    Q = _q(u, rb)
    assert list(Q[0, 0]) == [64, -127, 32, 0]
    assert list(Q[0, 2]) == [7, 2, -5, 0]
    assert r[0, 0] == F32(1) * (F32(1) / F32(127))
    assert r[0, 2] == F32(3) * (F32(1) / F32(7))


def test_decode_step_readout_does_not_depend_on_the_scheme():
    """The quantiser only decides what is stored: both schemes read out the same o and
    the same float32 state from the same packed input (lens decode-order paragraph)."""
    rng = np.random.default_rng(50)
    d, H = 128, 2
    rb = np.full((H, d), 6)
    om = rng.lognormal(size=(H, d)).astype(F32)
    S0 = rng.standard_normal((1, H, d, d)).astype(F32)
    u, r, c, piv = O.refit(S0, om, rb)
    q, k, v = (rng.standard_normal((1, H, d)).astype(F32) for _ in range(3))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    dec = np.full((1, H, d), F32(0.95))
    beta = np.full((1, H), F32(0.5))
    a = O.decode_step(u, r, c, piv, rb, om, q, k, v, dec, beta)
    b = O.decode_step(u, r, c, piv, rb, om, q, k, v, dec, beta, scheme="row_absmax")
    assert np.array_equal(a[4], b[4]) and np.array_equal(a[5], b[5])
    assert np.array_equal(b[0], O.absmax_quantise(b[5], rb)[0])


def test_absmax_all_pivot_head_stores_zero_scales():
    S = np.random.default_rng(60).standard_normal((1, 2, 128, 128)).astype(F32)
    rb = np.full((2, 128), 6)
    rb[1] = 16
    u, r, c, piv = O.absmax_quantise(S, rb)
    assert np.all(c[0, 0] == 1) and np.all(c[0, 1] == 0) and np.all(r[0, 1] == 0)
