"""Offline, lifetime-aware width allocation of a pool (the step before the decode path).

The method's offline stage (bloombook section 3, lifetime weight; section 4, the "time"
half: budgeted allocation and FP16 pivots; singularity-lens calibration paragraph):
every unit u (GDN head, KDA key row) gets a lifetime weight L_u from its mean
log-retention, a distortion D_u(b) for each candidate width b measured on calibration
states, and the widths that minimise sum_u L_u D_u(b_u) under a mean-bit budget, with
the riskiest units kept as FP16 pivots.

Every step runs in the library: the calibration states are quantised at each candidate
width by the quantise kernel (a pool of one uniform width), read back by the dequantise
kernel, and measured by the row-error kernel; lifetime weights, unit distortions and
the allocation are the library's host functions. This module only sequences the calls.
"""
from __future__ import annotations

import numpy as np

from . import stq

D = stq.D

CANDIDATES = {4: (2, 4, 6, 8), 6: (4, 6, 8)}   # candidate widths per nominal budget


def measure_distortions(kind, omega, states, cand_bits, stream=None):
    """D_u(b) for every unit and candidate: states [N, H, 128, 128] float32 on the GPU.
    Returns [n_units, n_cand] float64 (n_units = H for GDN, H*128 for KDA)."""
    import torch
    N, H = states.shape[0], states.shape[1]
    om = np.ascontiguousarray(omega, dtype=np.float32)
    slots = torch.arange(N, dtype=torch.int32, device=states.device)
    S_hat = torch.empty_like(states)
    err = torch.empty(N * H * D, dtype=torch.float32, device=states.device)
    n_units = H if kind == "gdn" else H * D
    out = np.empty((n_units, len(cand_bits)), np.float64)
    for ci, b in enumerate(cand_bits):
        ub = np.full(H if kind == "gdn" else H * D, b, np.uint8)
        pool = stq.Pool(kind, N, ub, om, device=states.device)
        pool.quantize_init(slots, states, stream)
        pool.dequantize(slots, S_hat, stream)
        pool.check(stream)
        stq.row_sq_error(states, S_hat, err, stream=stream)
        if stream is not None:
            stream.synchronize()
        else:
            torch.cuda.synchronize()
        out[:, ci] = stq.unit_distortion(kind, err.cpu().numpy().reshape(N, H, D), om)
        pool.close()
    return out


def allocate(kind, omega, states, ell_units, budget, pivot_frac=0.02, horizon=1024, cand_bits=None):
    """Widths per unit (GDN [H], KDA [H*128]; 16 = FP16 pivot) for a nominal budget of 4
    or 6 bits, from calibration states [N, H, 128, 128] on the GPU and each unit's mean
    log-retention ell_units. Returns (unit_bits uint8, details dict)."""
    cand = tuple(cand_bits) if cand_bits is not None else CANDIDATES[int(budget)]
    dist = measure_distortions(kind, omega, states, cand)
    ell = np.ascontiguousarray(ell_units, dtype=np.float64).reshape(-1)
    life = stq.lifetime_weights(ell, horizon)
    n_piv = int(round(pivot_frac * ell.size))
    bits = stq.allocate_bits(life, dist, cand, budget, n_piv)
    return bits, {"lifetime": life, "distortion": dist, "candidates": cand, "n_pivots": n_piv}


def in_head_distortions(kind, omega, states, unit_bits, cand_bits, stream=None):
    """D_u(b) of every KDA row measured inside the heads of a pool of widths unit_bits:
    the calibration states are quantised into that pool, and each row's error at every
    candidate width is taken with the column scales its head got
    (stq_row_error_at_widths). Returns [H*128, n_cand] float64."""
    import torch
    N, H = states.shape[0], states.shape[1]
    om = np.ascontiguousarray(omega, dtype=np.float32)
    slots = torch.arange(N, dtype=torch.int32, device=states.device)
    pool = stq.Pool(kind, N, unit_bits, om, device=states.device)
    pool.quantize_init(slots, states, stream)
    err = torch.empty((N, H, D, len(cand_bits)), dtype=torch.float32, device=states.device)
    pool.row_error_at_widths(slots, states, cand_bits, err, stream)
    pool.check(stream)
    e = err.cpu().numpy()
    pool.close()
    return np.stack([stq.unit_distortion(kind, np.ascontiguousarray(e[..., k]), om)
                     for k in range(len(cand_bits))], axis=1)


def allocate_in_head(kind, omega, states, ell_units, budget, pivot_frac=0.02, horizon=1024, rounds=3,
                     cand_bits=None, start="uniform"):
    """allocate(), then for per-row widths (KDA) up to `rounds` re-allocations on the
    rows' in-head distortions under the previous allocation (a row's width sets only the
    reach of its codes when its head shares column scales), stopping when no width
    changes. The first in-head distortions are taken under a pool of the budget width
    (start="uniform", which reaches the better widths) or under allocate()'s widths
    (start="allocated"). GDN heads have one width each, so
    the uniform-width distortions are already in-head ones and the first allocation
    stands. Returns (unit_bits, details)."""
    bits, info = allocate(kind, omega, states, ell_units, budget, pivot_frac, horizon, cand_bits)
    info["rounds"] = 0
    if kind == "gdn":
        return bits, info
    cand = info["candidates"]
    if start == "uniform":
        bits = np.full_like(bits, int(budget))
    for k in range(rounds):
        dist = in_head_distortions(kind, omega, states, bits, cand)
        new = stq.allocate_bits(info["lifetime"], dist, cand, budget, info["n_pivots"])
        info["rounds"] = k + 1
        info["distortion"] = dist
        if np.array_equal(new, bits):
            break
        bits = new
    return bits, info


def calibration_states(w, n_seq, steps, device="cuda"):
    """FP32 states after `steps` synthetic calibration steps from zero (FP32 step kernel)."""
    import torch
    from . import workload as W
    S = torch.zeros((n_seq, w.H, D, D), device=device)
    out = torch.empty((n_seq, w.H, D), device=device)
    for t in range(steps):
        x = W.calibration_step_inputs(w, t, n_seq)
        q, k, v, g, b = (torch.from_numpy(a).to(device) for a in (x.q, x.k, x.v, x.gate, x.beta))
        stq.fp32_decode_step(w.kind, S, q, k, v, g, b, out)
    return S


def main():
    """Allocate widths on synthetic calibration data, then compare the accumulated state
    error of the allocated pool with a uniform pool of the same mean width over paired
    FP32 / quantised runs (the pages' claim: lifetime-aware widths beat uniform ones)."""
    import argparse
    import json
    from . import build, diagnostics
    from . import workload as W
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--budget", type=int, default=6, choices=[4, 6])
    ap.add_argument("--sequences", type=int, default=32)
    ap.add_argument("--calib-steps", type=int, default=256)
    ap.add_argument("--eval-steps", type=int, default=1024)
    ap.add_argument("--eval-sequences", type=int, default=4)
    ap.add_argument("--in-head-rounds", type=int, default=3,
                    help="re-allocations of per-row (KDA) widths on in-head distortions (0: none)")
    ap.add_argument("--in-head-start", choices=["allocated", "uniform"], default="uniform",
                    help="pool whose column scales the first in-head distortions are taken under")
    a = ap.parse_args()
    build.build()
    w = W.WORKLOADS[a.workload]
    om = W.omega(w)
    S = calibration_states(w, a.sequences, a.calib_steps)
    bits, info = allocate_in_head(w.kind, om, S, W.calibration_log_retention(w), a.budget,
                                  rounds=a.in_head_rounds, start=a.in_head_start)
    del S
    hist = {str(b): int((bits == b).sum()) for b in sorted(set(bits.tolist()))}
    res = {"workload": w.name, "budget": a.budget, "calibration": f"{a.sequences} sequences x {a.calib_steps} steps",
           "evaluation": f"{a.eval_sequences} other sequences x {a.eval_steps} steps",
           "in_head_rounds": info["rounds"], "in_head_start": a.in_head_start,
           "widths": hist, "mean_bits_non_pivot": float(bits[bits != 16].mean()),
           "mean_bits_with_pivots": float(bits.mean())}
    uniform = np.full_like(bits, a.budget)
    for name, ub in (("allocated", bits), ("uniform", uniform)):
        r = diagnostics.error_lifetime(w, a.eval_sequences, a.eval_steps, scheme="stepquant", unit_bits=ub,
                                       first_seq=a.sequences)
        res[f"accumulated_sq_error_{name}"] = float(r["accumulated_sq_error"].sum())
    res["error_ratio_allocated_over_uniform"] = res["accumulated_sq_error_allocated"] / res["accumulated_sq_error_uniform"]
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
