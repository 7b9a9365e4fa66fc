"""Pins of the compact-scale variant of the oracle's quantisers (r and c stored as
binary16): the stored scales are binary16 values, the codes are the nearest codes for the
stored scales, the extra error over float32 scales is small, and the pool's bytes for
scales halve."""
import numpy as np
import pytest

from oracle import stq_oracle as O
from quantized_linear_attention_02_b200 import workload as W

F32 = np.float32


def _state(seed, H=3):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((2, H, 128, 128)).astype(F32)
    S[:, :, 5, :] *= 10
    S[:, :, :, 7] *= 10
    om = rng.lognormal(size=(H, 128)).astype(F32)
    return S, om


def _is_half(x):
    return np.array_equal(np.asarray(x, F32).astype(np.float16).astype(F32), np.asarray(x, F32))


@pytest.mark.parametrize("bits", [2, 4, 6, 8])
@pytest.mark.parametrize("scheme", ["stepquant", "row_absmax"])
def test_scale16_scales_are_half_and_codes_fit_them(bits, scheme):
    S, om = _state(bits)
    rb = np.full((3, 128), bits)
    if scheme == "stepquant":
        u, r, c, _ = O.refit(S, om, rb, scale16=True)
    else:
        u, r, c, _ = O.absmax_quantise(S, rb, scale16=True)
    assert _is_half(r) and _is_half(c)
    Q = u - O.bias_of(rb)[..., None]
    qm = 2 ** (bits - 1) - 1
    # nearest code for the stored scales wherever the code is not at the clamp
    x = (S.astype(np.float64) / r.astype(np.float64)[..., :, None]) / c.astype(np.float64)[..., None, :]
    inner = np.abs(Q) < qm
    assert np.all(np.abs(x - Q)[inner] <= 0.5 + 1e-5)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_scale16_costs_little_accuracy(bits):
    S, om = _state(20 + bits)
    rb = np.full((3, 128), bits)
    e = {}
    for s16 in (False, True):
        u, r, c, piv = O.refit(S, om, rb, scale16=s16)
        e[s16] = np.linalg.norm(O.dequantize(u, r, c, piv, rb).astype(np.float64) - S)
    assert e[True] <= 1.02 * e[False]


def test_scale16_pool_image_round_trip_and_bytes():
    w = W.WORKLOADS[1]
    rb = W.row_bits(w)
    S, _ = _state(5, H=w.H)
    u, r, c, piv = O.refit(S[:1], W.omega(w), rb, scale16=True)
    L = O.Layout(rb)
    img = O.Pool(L, 2, scale16=True)
    img.write_heads([1], u, r, c, piv)
    u2, r2, c2, p2 = img.read_heads([1])
    assert np.array_equal(u2, u) and np.array_equal(r2, r) and np.array_equal(c2, c)
    assert img.scales.nbytes * 2 == O.Pool(L, 2).scales.nbytes
