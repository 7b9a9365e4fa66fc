"""GPU parity of the offline width allocation: the row-error kernel against the oracle's
tree sums, and the whole allocation (quantise each candidate width, dequantise, measure,
weigh by lifetime, allocate) against the oracle's pipeline on the same synthetic
calibration states."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from oracle import stq_alloc as A  # noqa: E402
from oracle import stq_oracle as O  # noqa: E402
from quantized_linear_attention_02_b200 import build, calibrate, stq  # noqa: E402
from quantized_linear_attention_02_b200 import workload as W  # noqa: E402

D = 128
F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    build.build()
    stq.lib()


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def test_row_sq_error_bit_exact_and_accumulate():
    rng = np.random.default_rng(0)
    S = rng.standard_normal((5, 3, D, D)).astype(F32)
    Sh = (S + rng.standard_normal(S.shape).astype(F32) * F32(0.03)).astype(F32)
    err = torch.empty(5 * 3 * D, device="cuda")
    stq.row_sq_error(dev(S), dev(Sh), err)
    ref = A.row_sq_error(S, Sh).reshape(-1)
    assert np.array_equal(err.cpu().numpy(), ref)
    stq.row_sq_error(dev(S), dev(S * F32(0.5)), err, accumulate=True)
    ref2 = (ref + A.row_sq_error(S, S * F32(0.5)).reshape(-1)).astype(F32)
    torch.cuda.synchronize()
    assert np.array_equal(err.cpu().numpy(), ref2)


def _calibration_states(w, n_seq, steps):
    """FP32 runs from zero over the synthetic calibration inputs: oracle on the CPU and
    the FP32 step kernel on the GPU (bit-exact with each other)."""
    S = np.zeros((n_seq, w.H, D, D), F32)
    Sg = torch.zeros((n_seq, w.H, D, D), device="cuda")
    out = torch.empty((n_seq, w.H, D), device="cuda")
    for t in range(steps):
        x = W.calibration_step_inputs(w, t, n_seq)
        S, _ = O.fp32_step(S, x.q, x.k, x.v, O.gate_rows(x.gate, w.kind, D), x.beta)
        stq.fp32_decode_step(w.kind, Sg, dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
    torch.cuda.synchronize()
    assert np.array_equal(Sg.cpu().numpy(), S)
    return S, Sg


@pytest.mark.parametrize("widx,budget,n_seq,steps", [(1, 6, 4, 32), (1, 4, 4, 32), (2, 4, 2, 24)])
def test_allocation_pipeline_matches_oracle(widx, budget, n_seq, steps):
    w = W.WORKLOADS[widx]
    om = W.omega(w)
    ell = W.calibration_log_retention(w)
    S, Sg = _calibration_states(w, n_seq, steps)
    bits, info = calibrate.allocate(w.kind, om, Sg, ell, budget, pivot_frac=0.02)
    cand = calibrate.CANDIDATES[budget]
    # the oracle's pipeline on the same states
    dist = np.empty((w.n_units, len(cand)))
    for ci, b in enumerate(cand):
        rb = np.full((w.H, D), b)
        u, r, c, piv = O.refit(S, om, rb)
        e = A.row_sq_error(S, O.dequantize(u, r, c, piv, rb))
        dist[:, ci] = A.unit_distortion(w.kind, e, om)
    # codes may differ by one at a rounding boundary (at most 1e-5 of them), so the
    # distortions agree to rounding, not bit for bit
    assert np.allclose(info["distortion"], dist, rtol=1e-4, atol=0)
    life = A.lifetime_weight(ell.reshape(-1))
    ref = A.allocate(life, info["distortion"], cand, budget, info["n_pivots"])
    assert np.array_equal(bits.astype(np.int64), ref)
    ref_or = A.allocate(life, dist, cand, budget, info["n_pivots"])
    assert np.mean(bits.astype(np.int64) == ref_or) >= 0.99
    # the allocation spends the budget on the units that keep errors longest
    rest = bits != 16
    assert bits[rest].astype(int).mean() <= budget
    lo = np.argsort(life)[: life.size // 4]
    hi = np.argsort(life)[-life.size // 4:]
    assert bits[hi][bits[hi] != 16].mean() >= bits[lo][bits[lo] != 16].mean()


@pytest.mark.parametrize("widx", [1, 2])
def test_error_lifetime_diagnostic_matches_oracle(widx):
    """A short paired run (FP32 vs uniform INT6 absmax, shared inputs): the GPU's
    accumulated per-unit squared state error equals the oracle's to chain tolerance."""
    from quantized_linear_attention_02_b200 import diagnostics
    w = W.WORKLOADS[widx]
    n_seq, steps = 2, 8
    r = diagnostics.error_lifetime(w, n_seq=n_seq, steps=steps, bits=6)
    rb = np.full((w.H, D), 6)
    S = np.zeros((n_seq, w.H, D, D), F32)
    u, rr, c, piv = O.absmax_quantise(S, rb)
    acc = np.zeros((n_seq, w.H, D), F32)
    for t in range(steps):
        x = W.calibration_step_inputs(w, t, n_seq)
        dec = O.gate_rows(x.gate, w.kind, D)
        u, rr, c, piv, _, _ = O.decode_step(u, rr, c, piv, rb, W.omega(w), x.q, x.k, x.v, dec, x.beta,
                                            scheme="row_absmax")
        S, _ = O.fp32_step(S, x.q, x.k, x.v, dec, x.beta)
        acc = (acc + A.row_sq_error(O.dequantize(u, rr, c, piv, rb), S)).astype(F32)
    rows = acc.astype(np.float64).sum(axis=0)
    err = rows.sum(axis=1) if w.kind == "gdn" else rows.reshape(-1)
    assert np.allclose(r["accumulated_sq_error"], err, rtol=1e-3, atol=1e-30)
    assert np.allclose(r["half_life"], np.log(0.5) / W.calibration_log_retention(w).reshape(-1))


@pytest.mark.parametrize("scale_bits", [32, 16])
def test_row_error_at_widths_matches_oracle(scale_bits):
    """The in-head row errors (stq_row_error_at_widths) equal the oracle's bit for bit:
    a KDA pool of mixed per-row widths with a pivot row, quantised from random states."""
    rng = np.random.default_rng(5)
    H, N = 3, 4
    S = (rng.standard_normal((N, H, D, D)) * rng.lognormal(0, 1, (N, H, D, 1))).astype(F32)
    om = rng.lognormal(0, 1, (H, D)).astype(F32)
    rb = rng.choice([2, 4, 6, 8], size=(H, D))
    rb[1, 9] = 16
    pool = stq.Pool("kda", N + 2, rb.reshape(-1).astype(np.uint8), om, scale_bits=scale_bits)
    slots = torch.tensor([2, 0, 5, 3], dtype=torch.int32, device="cuda")
    Sg = dev(S)
    pool.quantize_init(slots, Sg)
    cand = (2, 4, 6, 8)
    err = torch.empty((N, H, D, len(cand)), device="cuda")
    pool.row_error_at_widths(slots, Sg, cand, err)
    pool.check()
    c = pool.scales_view()[slots.long(), :, 1].float().cpu().numpy()
    ref = A.row_error_at_widths(S, c, om, cand, scale16=scale_bits == 16)
    assert np.array_equal(err.cpu().numpy(), ref)
