"""Shared helpers of the parity tests: oracle-side state preparation, copying an
oracle pool image into the library's buffers, and the comparison rules."""
from __future__ import annotations

import functools

import numpy as np

from oracle import stq_oracle as O
from quantized_linear_attention_02_b200 import workload as W

F32 = np.float32
D = 128

# Tolerances (stated by the decode-step contract): codes equal except elements whose
# exact x lies within 1e-6 relative of a rounding boundary, at most 1e-5 of codes and
# each off by one; readout relative L2 <= 1e-4; dequantised states after 64 chained
# steps relative L2 <= 1e-3.
BOUNDARY_REL = 1e-6
MAX_FLIP_FRAC = 1e-5
OUT_REL_L2 = 1e-4
CHAIN_REL_L2 = 1e-3


def unit_bits_rows(w):
    return W.unit_bits(w), W.row_bits(w)


@functools.lru_cache(maxsize=None)
def warm_state(widx: int, reqs: tuple, steps: int | None = None) -> np.ndarray:
    """Initial float32 states [len(reqs), H, d, d] of the given requests: FP32 warm-up
    steps from zero (oracle arithmetic), then the x10 outlier rows."""
    w = W.WORKLOADS[widx]
    steps = w.warmup_steps if steps is None else steps
    S = np.zeros((len(reqs), w.H, D, D), F32)
    for t in range(steps):
        parts = [W.step_inputs(w, "warmup", t, b, b + 1) for b in reqs]
        x = _cat(parts)
        S, _ = O.fp32_step(S, x.q, x.k, x.v, O.gate_rows(x.gate, w.kind, D), x.beta)
    return W.scale_outlier_rows(S, w)


def warm_states(widx: int, reqs, steps: int | None = None) -> np.ndarray:
    """warm_state of several requests, one request per worker process (the warm-up of
    each request is independent of the others). The pool is started with `spawn`, so it
    is safe after CUDA is initialised; the workers run NumPy only."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    reqs = [int(b) for b in reqs]
    n = min(len(reqs), len(os.sched_getaffinity(0)))
    if n <= 1:
        return warm_state(widx, tuple(reqs), steps)
    with cf.ProcessPoolExecutor(n, mp_context=mp.get_context("spawn")) as ex:
        parts = list(ex.map(warm_state, [widx] * len(reqs), [(b,) for b in reqs], [steps] * len(reqs)))
    return np.concatenate(parts, 0)


def oracle_chain(widx: int, b: int, state, t0: int, steps: int, keep_states=()):
    """The oracle's decode steps t0 .. t0+steps-1 of request b from the packed state
    (u, r, c, piv) of that request ([1, H, ...] arrays). Returns (readouts [steps, H, d],
    final (u, r, c, piv), {t: dequantised state after step t for t in keep_states})."""
    w = W.WORKLOADS[widx]
    rb, om = W.row_bits(w), W.omega(w)
    u, r, c, piv = state
    outs, kept = [], {}
    for t in range(t0, t0 + steps):
        x = W.step_inputs(w, "decode", t, b, b + 1)
        u, r, c, piv, o, _ = O.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v,
                                           O.gate_rows(x.gate, w.kind, D), x.beta)
        outs.append(o[0])
        if t + 1 - t0 in keep_states:
            kept[t + 1 - t0] = O.dequantize(u, r, c, piv, rb)[0]
    return np.stack(outs), (u, r, c, piv), kept


def oracle_chains(widx: int, reqs, states, t0: int, steps: int, keep_states=()):
    """oracle_chain of several requests, one per spawn-started worker process (the
    chains are independent). states: (u, r, c, piv) with a leading request axis."""
    import concurrent.futures as cf
    import multiprocessing as mp
    import os
    reqs = [int(b) for b in reqs]
    per = [tuple(a[n:n + 1] for a in states) for n in range(len(reqs))]
    n = min(len(reqs), len(os.sched_getaffinity(0)))
    if n <= 1:
        return [oracle_chain(widx, b, st, t0, steps, keep_states) for b, st in zip(reqs, per)]
    with cf.ProcessPoolExecutor(n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(oracle_chain, [widx] * len(reqs), reqs, per, [t0] * len(reqs),
                           [steps] * len(reqs), [tuple(keep_states)] * len(reqs)))


# Reported (not gated) measurements of the GPU parity tests, printed at the end of the
# run by tests/conftest.py: {name: text}.
REPORTS: dict = {}


def _cat(parts):
    return W.StepInputs(*[np.concatenate([getattr(p, n) for p in parts], 0)
                          for n in ("q", "k", "v", "gate", "beta")])


def inputs_for(w, phase, t, reqs):
    return _cat([W.step_inputs(w, phase, t, b, b + 1) for b in reqs])


def write_oracle_state(pool, layout, slots, u, r, c, piv):
    """Put an oracle-packed state into the library pool's buffers (host image ->
    device copy of the same bytes)."""
    import torch
    img = O.Pool(layout, pool.n_slots, scale16=getattr(pool, "scale_bits", 32) == 16)
    img.write_heads(list(range(len(slots))), u, r, c, piv)   # rows 0..n-1 of the image
    for n, s in enumerate(slots):
        pool.codes_view()[s].copy_(torch.from_numpy(img.codes[n]))
        pool.scales_view()[s].copy_(torch.from_numpy(img.scales[n]))
        if layout.n_pivot_rows:
            pool.pivots_view()[s].copy_(torch.from_numpy(img.pivots[n]))


def read_pool_state(pool, layout, slots):
    """Read the library pool's bytes for the given slots and decode them with the
    oracle's unpacker: (u, r, c, piv)."""
    img = O.Pool(layout, len(slots), scale16=getattr(pool, "scale_bits", 32) == 16)
    for n, s in enumerate(slots):
        img.codes[n] = pool.codes_view()[s].cpu().numpy()
        img.scales[n] = pool.scales_view()[s].cpu().numpy()
        if layout.n_pivot_rows:
            img.pivots[n] = pool.pivots_view()[s].cpu().numpy()
    return img.read_heads(list(range(len(slots))))


def near_boundary(X, r, c, row_bits):
    """Elements whose exact quantiser argument x = (X_ij / r_i) / c_j (as the rule
    evaluates it) lies within BOUNDARY_REL relative of a half-integer."""
    inv_r = O._recip(r)
    y = (np.asarray(X, F32) * inv_r[..., :, None]).astype(np.float64)
    x = np.abs(y * O._recip(c).astype(np.float64)[..., None, :])
    return np.abs(x - np.floor(x) - 0.5) <= BOUNDARY_REL * x


# Codes compared per workload during the session: {workload: [codes that differ, codes
# compared]}; tests/conftest.py prints it at the end of the run.
FLIPS: dict = {}


def record_flips(config, n_diff, n_codes):
    tot = FLIPS.setdefault(config, [0, 0])
    tot[0] += int(n_diff)
    tot[1] += int(n_codes)


def compare_codes(u_gpu, u_or, X, r_or, c_or, row_bits, what="", config="other"):
    """Assert the code rule; return the number of (allowed) mismatches. Every comparison
    is added to FLIPS under `config`."""
    nonpiv = np.broadcast_to((np.asarray(row_bits) != O.PIVOT_BITS)[..., None], np.shape(u_or))
    diff = (u_gpu != u_or) & nonpiv
    n = int(diff.sum())
    record_flips(config, n, int(nonpiv.sum()))
    if n:
        nb = near_boundary(X, r_or, c_or, row_bits)
        assert np.all(np.abs(u_gpu - u_or)[diff] == 1), f"{what}: a code differs by more than 1"
        assert np.all(nb[diff]), f"{what}: {n} code(s) differ away from a rounding boundary"
        assert n <= MAX_FLIP_FRAC * nonpiv.sum(), f"{what}: {n} boundary flips exceed 1e-5"
    return n


C_REL_WITH_FLIPS = 1e-5


def check_scales(r_gpu, r_or, c_gpu, c_or, flips, what="", c_rel=C_REL_WITH_FLIPS):
    """Scales of a step (or a quantisation) from an identical input: r is formed before
    any code is decided, so it matches bit for bit whatever happened to the codes; c
    matches bit for bit when no code differs, else within c_rel relative (binary16
    scales: pass one binary16 step, 2^-10)."""
    assert np.array_equal(r_gpu, r_or), f"{what}: row scales differ"
    if flips == 0:
        assert np.array_equal(c_gpu, c_or), f"{what}: column scales differ"
    else:
        c_or = np.asarray(c_or, np.float64)
        rel = np.abs(np.asarray(c_gpu, np.float64) - c_or) / np.maximum(np.abs(c_or), 1e-300)
        assert rel.max() <= c_rel, f"{what}: column scales differ by {rel.max():.3g} relative"


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def per_vector_rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    num = np.linalg.norm(a - b, axis=-1)
    den = np.maximum(np.linalg.norm(b, axis=-1), 1e-300)
    return num / den
