"""Seeded synthetic workloads for the packed Delta-rule state decode step.

This module only draws random numbers and shapes them into inputs: allocation
maps, row-influence weights, outlier index sets and per-step (q, k, v, gate, beta)
tensors. It holds none of the method's arithmetic (no state update, no
quantisation, no packing); both the CUDA path and the CPU oracle consume what it
produces.

Workloads follow the decode setting of "STEPQuant: When and Where Errors Matter in
Delta-Rule Recurrent State Quantization" (arXiv 2609.38169) as the pages describe it:
  * GDN units are whole heads, KDA units are key rows (singularity-lens page,
    "GDN and KDA" paragraph; ai-trend page, Method);
  * allocation candidates {4,6,8} for the nominal 6-bit budget and {2,4,6,8} for the
    nominal 4-bit budget, plus a few FP16 pivot units (singularity-lens page,
    calibration paragraph; bloombook page, section 4);
  * row and column outliers persist through decoding (bloombook page, section 3,
    Figure 2 discussion).
The random recipe itself (distributions, fractions, outlier factor) is the workload
definition each config states.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

D = 128                 # d_k = d_v
PIVOT_BITS = 16         # unit width marker for an FP16 pivot unit
OUTLIER_FACTOR = 10.0
OUTLIER_FRAC = 0.05


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    kind: str                 # "gdn" or "kda"
    B: int
    H: int
    alloc: tuple              # ((bits, fraction), ...) in listed order
    pivot_frac: float
    omega: str                # "ones" or "lognormal"
    outliers: bool
    steps: int
    warmup_steps: int = 256
    d: int = D
    gate_low: float = -0.2
    gate_high: float = -0.001

    @property
    def n_units(self) -> int:
        return self.H if self.kind == "gdn" else self.H * self.d


WORKLOADS = [
    Workload(0, "gdn_b1_h4_uniform8", "gdn", 1, 4, ((8, 1.0),), 0.0, "ones", False, 16),
    Workload(1, "gdn_b32_h48_nominal6", "gdn", 32, 48, ((4, 0.2), (6, 0.5), (8, 0.3)),
             0.02, "lognormal", True, 64),
    Workload(2, "kda_b64_h32_nominal4", "kda", 64, 32,
             ((2, 0.15), (4, 0.55), (6, 0.2), (8, 0.1)), 0.02, "lognormal", True, 64,
             gate_low=-0.5, gate_high=-0.0005),
    Workload(3, "gdn_b512_h48_nominal6", "gdn", 512, 48, ((4, 0.2), (6, 0.5), (8, 0.3)),
             0.02, "lognormal", True, 1),
    Workload(4, "kda_b512_h32_nominal6", "kda", 512, 32, ((4, 0.2), (6, 0.5), (8, 0.3)),
             0.02, "lognormal", True, 1024, gate_low=-0.5, gate_high=-0.0005),
]


def _streams(index: int):
    """Six independent sub-streams per workload: allocation, omega, outliers,
    warm-up inputs, step inputs, parity sample."""
    ss = np.random.SeedSequence(index)
    return [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(6)]


def unit_counts(n_units: int, alloc, pivot_frac: float):
    """Integer unit counts per width: pivots = round(frac * n); the rest split by
    largest remainder, ties to the earlier listed width."""
    n_piv = int(round(pivot_frac * n_units))
    rest = n_units - n_piv
    raw = [f * rest for _, f in alloc]
    base = [int(math.floor(x)) for x in raw]
    left = rest - sum(base)
    order = sorted(range(len(raw)), key=lambda i: (-(raw[i] - base[i]), i))
    for i in order[:left]:
        base[i] += 1
    return n_piv, [(b, n) for (b, _), n in zip(alloc, base)]


def unit_bits(w: Workload) -> np.ndarray:
    """Per-unit widths (2/4/6/8, or 16 for a pivot): GDN [H], KDA [H*d] (uint8).
    Widths are handed out over a seeded permutation of the units."""
    rng = _streams(w.index)[0]
    n = w.n_units
    n_piv, counts = unit_counts(n, w.alloc, w.pivot_frac)
    seq = [PIVOT_BITS] * n_piv
    for b, c in counts:
        seq += [b] * c
    perm = rng.permutation(n)
    out = np.empty(n, dtype=np.uint8)
    out[perm] = np.asarray(seq, dtype=np.uint8)
    return out


def row_bits(w: Workload) -> np.ndarray:
    """Widths expanded per key row: [H, d] uint8."""
    ub = unit_bits(w)
    if w.kind == "gdn":
        return np.repeat(ub[:, None], w.d, axis=1)
    return ub.reshape(w.H, w.d)


def omega(w: Workload) -> np.ndarray:
    """Static row-influence weights [H, d] float32 (> 0), shared by all requests."""
    if w.omega == "ones":
        return np.ones((w.H, w.d), dtype=np.float32)
    rng = _streams(w.index)[1]
    return rng.lognormal(0.0, 1.0, size=(w.H, w.d)).astype(np.float32)


def outlier_sets(w: Workload):
    """Per head, the rows and the columns that carry x10 outliers: two [H, m] int
    arrays (m = 5% of d rounded down), or empty arrays when the workload has none."""
    m = int(OUTLIER_FRAC * w.d)
    if not w.outliers:
        z = np.zeros((w.H, 0), dtype=np.int64)
        return z, z
    rng = _streams(w.index)[2]
    rows = np.stack([np.sort(rng.choice(w.d, m, replace=False)) for _ in range(w.H)])
    cols = np.stack([np.sort(rng.choice(w.d, m, replace=False)) for _ in range(w.H)])
    return rows, cols


@dataclass
class StepInputs:
    q: np.ndarray       # [B, H, d] float32, unit L2 norm
    k: np.ndarray       # [B, H, d] float32, unit L2 norm
    v: np.ndarray       # [B, H, d] float32
    gate: np.ndarray    # GDN [B, H], KDA [B, H, d]; multiplicative retention alpha
    beta: np.ndarray    # [B, H] float32 in (0, 1)


def _draw(rng, w: Workload, nb: int, col_out) -> StepInputs:
    H, d = w.H, w.d
    q = rng.standard_normal((nb, H, d))
    k = rng.standard_normal((nb, H, d))
    v = rng.standard_normal((nb, H, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    if col_out.shape[1]:
        hh = np.arange(H)[:, None]
        v[:, hh, col_out] *= OUTLIER_FACTOR
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((nb, H))))
    gshape = (nb, H) if w.kind == "gdn" else (nb, H, d)
    ell = rng.uniform(w.gate_low, w.gate_high, size=gshape)
    gate = np.exp(ell)      # host-side exp in float64, rounded once to float32
    f = np.float32
    return StepInputs(q.astype(f), k.astype(f), v.astype(f), gate.astype(f), beta.astype(f))


def step_inputs(w: Workload, phase: str, step: int, b0: int = 0, b1: int | None = None) -> StepInputs:
    """Inputs of one decode step for requests [b0, b1). phase is "warmup" or "decode".
    Each (phase, step, request) gets its own counter-derived stream, so any subset of
    requests is reproducible on its own."""
    b1 = w.B if b1 is None else b1
    _, cols = outlier_sets(w)
    tag = 3 if phase == "warmup" else 4
    parts = []
    for b in range(b0, b1):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.index, tag, step, b])))
        parts.append(_draw(rng, w, 1, cols))
    cat = lambda name: np.concatenate([getattr(p, name) for p in parts], axis=0)
    return StepInputs(cat("q"), cat("k"), cat("v"), cat("gate"), cat("beta"))


def slot_of_request(b: int) -> int:
    """Requests use spread slots of a (5B+1)-slot pool, as the serving stack the pages
    describe reserves five state slots per request (zhichai page, forum reply)."""
    return 5 * b + 1


def n_slots(B: int) -> int:
    return 5 * B + 1


def parity_sample(w: Workload, n: int) -> np.ndarray:
    """Seeded sample of n request indices (sorted) for checking large workloads."""
    rng = _streams(w.index)[5]
    return np.sort(rng.choice(w.B, size=min(n, w.B), replace=False))


def scale_outlier_rows(S: np.ndarray, w: Workload) -> np.ndarray:
    """Multiply each head's outlier rows of an initial state [B, H, d, d] by the
    outlier factor (applied once, after warm-up)."""
    rows, _ = outlier_sets(w)
    if rows.shape[1] == 0:
        return S
    S = S.copy()
    hh = np.arange(w.H)[:, None]
    S[:, hh, rows, :] *= np.float32(OUTLIER_FACTOR)
    return S


def torch_step_inputs(w: Workload, B: int, generator, device="cuda"):
    """The same input recipe drawn with torch's device RNG (fast, for large batches
    whose exact values no oracle needs): returns q, k, v, gate, beta tensors."""
    import torch
    H, d = w.H, w.d
    g = generator
    q = torch.nn.functional.normalize(torch.randn((B, H, d), device=device, generator=g), dim=-1)
    k = torch.nn.functional.normalize(torch.randn((B, H, d), device=device, generator=g), dim=-1)
    v = torch.randn((B, H, d), device=device, generator=g)
    _, cols = outlier_sets(w)
    if cols.shape[1]:
        scale = torch.ones((H, d), device=device)
        hh = torch.arange(H, device=device)[:, None]
        scale[hh, torch.as_tensor(cols, device=device)] = OUTLIER_FACTOR
        v = v * scale
    gshape = (B, H) if w.kind == "gdn" else (B, H, d)
    gate = torch.exp(torch.empty(gshape, device=device, dtype=torch.float64)
                     .uniform_(w.gate_low, w.gate_high, generator=g)).float()
    beta = torch.sigmoid(torch.randn((B, H), device=device, generator=g))
    return q.contiguous(), k.contiguous(), v.contiguous(), gate.contiguous(), beta.contiguous()


def torch_scale_outlier_rows(S, w: Workload):
    """Device version of scale_outlier_rows for a [B, H, d, d] tensor (in place)."""
    import torch
    rows, _ = outlier_sets(w)
    if rows.shape[1] == 0:
        return S
    hh = torch.arange(w.H, device=S.device)[:, None]
    S[:, hh, torch.as_tensor(rows, device=S.device), :] *= OUTLIER_FACTOR
    return S


# ---------------------------------------------------------------------------------
# synthetic calibration data for the offline width allocation
# ---------------------------------------------------------------------------------
CALIB_JITTER = 0.1      # per-step log-retention = mean * (1 + U(-0.1, 0.1))


def calibration_log_retention(w: Workload) -> np.ndarray:
    """Mean log-retention of every unit in the synthetic calibration data (GDN [H],
    KDA [H, d], float64), drawn once per unit from U(gate_low, gate_high) so that units
    differ in memory length (half-lives ln 0.5 / l from a few steps to several
    hundred). The pages estimate it from 32 WikiText-2 segments, which are not here."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.index, 7])))
    shape = (w.H,) if w.kind == "gdn" else (w.H, w.d)
    return rng.uniform(w.gate_low, w.gate_high, size=shape)


def calibration_step_inputs(w: Workload, step: int, n_seq: int, first_seq: int = 0) -> StepInputs:
    """Inputs of calibration step `step` for sequences first_seq .. first_seq + n_seq - 1:
    q, k, v, beta drawn as decode inputs; the gate of unit u is exp(l_u (1 + e)),
    e ~ U(-CALIB_JITTER, CALIB_JITTER) per (sequence, unit), so its mean log-retention
    is l_u."""
    _, cols = outlier_sets(w)
    ell_u = calibration_log_retention(w)
    parts = []
    for s in range(first_seq, first_seq + n_seq):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.index, 8, step, s])))
        x = _draw(rng, w, 1, cols)
        jit = rng.uniform(-CALIB_JITTER, CALIB_JITTER, size=ell_u.shape)
        gate = np.exp(ell_u * (1.0 + jit))[None].astype(np.float32)
        parts.append(StepInputs(x.q, x.k, x.v, gate, x.beta))
    cat = lambda name: np.concatenate([getattr(p, name) for p in parts], axis=0)
    return StepInputs(cat("q"), cat("k"), cat("v"), cat("gate"), cat("beta"))
