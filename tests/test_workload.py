"""The seeded workload generator: determinism and unit counts per config."""
import numpy as np
import pytest

from quantized_linear_attention_02_b200 import workload as W


def test_unit_counts_per_config():
    # largest-remainder split of the non-pivot units; pivots = round(2% of units)
    assert W.unit_counts(48, W.WORKLOADS[1].alloc, 0.02) == (1, [(4, 9), (6, 24), (8, 14)])
    assert W.unit_counts(4096, W.WORKLOADS[2].alloc, 0.02) == (82, [(2, 602), (4, 2208), (6, 803), (8, 401)])
    assert W.unit_counts(4096, W.WORKLOADS[4].alloc, 0.02) == (82, [(4, 803), (6, 2007), (8, 1204)])
    assert W.unit_counts(4, W.WORKLOADS[0].alloc, 0.0) == (0, [(8, 4)])


@pytest.mark.parametrize("w", W.WORKLOADS, ids=lambda w: w.name)
def test_allocation_is_seeded_and_complete(w):
    a, b = W.unit_bits(w), W.unit_bits(w)
    assert np.array_equal(a, b)
    n_piv, counts = W.unit_counts(w.n_units, w.alloc, w.pivot_frac)
    assert int((a == 16).sum()) == n_piv
    for bits, n in counts:
        assert int((a == bits).sum()) == n
    rb = W.row_bits(w)
    assert rb.shape == (w.H, w.d)


def test_step_inputs_subset_reproducible():
    w = W.WORKLOADS[1]
    full = W.step_inputs(w, "decode", 3, 0, 6)
    part = W.step_inputs(w, "decode", 3, 2, 4)
    for name in ("q", "k", "v", "gate", "beta"):
        assert np.array_equal(getattr(full, name)[2:4], getattr(part, name))
    assert np.allclose(np.linalg.norm(full.q, axis=-1), 1, atol=1e-6)
    assert np.all((full.gate > np.exp(-0.2) - 1e-7) & (full.gate < 1))
    kda = W.step_inputs(W.WORKLOADS[2], "warmup", 0, 0, 2)
    assert kda.gate.shape == (2, 32, 128)


def test_outlier_columns_scaled():
    w = W.WORKLOADS[1]
    rows, cols = W.outlier_sets(w)
    assert rows.shape == (48, 6) and cols.shape == (48, 6)
    x = W.step_inputs(w, "decode", 0, 0, 64)
    h = 5
    mask = np.zeros(128, bool); mask[cols[h]] = True
    assert np.std(x.v[:, h, mask]) > 5 * np.std(x.v[:, h, ~mask])


def test_parallel_warm_states_equal_serial():
    # the spawn-pool warm-up the full-size parity tests use gives the serial states
    import stq_testlib as T
    w = W.WORKLOADS[2]
    reqs = [3, 17, 40]
    a = T.warm_states(w.index, reqs, steps=6)
    b = T.warm_state(w.index, tuple(reqs), 6)
    assert a.dtype == np.float32 and np.array_equal(a, b)
