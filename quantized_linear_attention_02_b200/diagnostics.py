"""Error-lifetime diagnostic: does a unit's memory length predict how much state error it
accumulates under uniform quantisation?

The pages' mechanism check (bloombook section 3; singularity-lens evaluation-setup
paragraph; ai-trend review, Results): an FP32 run and a uniform INT6 run share their
inputs for 2,046 updates, and the Spearman correlation between each unit's gate half-life
and its accumulated squared state error is about 0.80. Here the runs are synthetic (the
pages use 4 C4 sequences through the real models, which are not available): the
calibration inputs give every unit its own mean log-retention l_u, half-life
ln(0.5) / l_u, and both chains run on the GPU through the library:
  * FP32 chain: the FP32-state step kernel;
  * INT6 chain: a pool of uniform width b with the symmetric per-key-row absmax
    quantiser (the pages' uniform baseline), decode step kernel;
  * after every step the INT6 state is dequantised and the row-error kernel adds
    sum_j (S_int6 - S_fp32)^2 of every key row into a float32 accumulator.
Units are GDN heads (their rows summed) or KDA key rows.

Run: python -m quantized_linear_attention_02_b200.diagnostics --workload 1 --steps 2046
"""
from __future__ import annotations

import argparse
import json

import numpy as np

from . import stq
from . import workload as W

D = stq.D


def error_lifetime(w, n_seq=4, steps=2046, bits=6, scheme="row_absmax", device="cuda", unit_bits=None,
                   first_seq=0):
    """Returns dict with per-unit half-life, accumulated squared error and Spearman rho.
    unit_bits (GDN [H], KDA [H*128]) overrides the uniform width `bits`; the runs use
    calibration sequences first_seq .. first_seq + n_seq - 1."""
    import torch
    from scipy.stats import spearmanr
    H = w.H
    n_units = H if w.kind == "gdn" else H * D
    ub = np.full(n_units, bits, np.uint8) if unit_bits is None else np.asarray(unit_bits, np.uint8)
    pool = stq.Pool(w.kind, n_seq, ub, W.omega(w), device=device, scheme=scheme)
    slots = torch.arange(n_seq, dtype=torch.int32, device=device)
    S = torch.zeros((n_seq, H, D, D), device=device)
    pool.quantize_init(slots, S)
    S_hat = torch.empty_like(S)
    acc = torch.zeros(n_seq * H * D, device=device)
    o_q = torch.empty((n_seq, H, D), device=device)
    o_f = torch.empty_like(o_q)
    for t in range(steps):
        x = W.calibration_step_inputs(w, t, n_seq, first_seq)
        q, k, v, g, b = (torch.from_numpy(a).to(device) for a in (x.q, x.k, x.v, x.gate, x.beta))
        pool.decode_step(slots, q, k, v, g, b, o_q)
        stq.fp32_decode_step(w.kind, S, q, k, v, g, b, o_f)
        pool.dequantize(slots, S_hat)
        stq.row_sq_error(S_hat, S, acc, accumulate=True)
    pool.check()
    rows = acc.view(n_seq, H, D).cpu().numpy().astype(np.float64).sum(axis=0)   # [H, D]
    err = rows.sum(axis=1) if w.kind == "gdn" else rows.reshape(-1)
    ell = W.calibration_log_retention(w).reshape(-1)
    half_life = np.log(0.5) / ell
    rho = float(spearmanr(half_life, err).correlation)
    return {"workload": w.name, "kind": w.kind, "units": int(n_units), "sequences": n_seq,
            "steps": steps, "bits": bits, "scheme": scheme, "spearman_half_life_vs_error": rho,
            "half_life": half_life, "accumulated_sq_error": err}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2046)
    ap.add_argument("--sequences", type=int, default=4)
    ap.add_argument("--bits", type=int, default=6)
    ap.add_argument("--scheme", default="row_absmax", choices=["row_absmax", "stepquant"])
    a = ap.parse_args()
    from . import build
    build.build()
    r = error_lifetime(W.WORKLOADS[a.workload], a.sequences, a.steps, a.bits, a.scheme)
    hl, er = r.pop("half_life"), r.pop("accumulated_sq_error")
    q = np.quantile(hl, [0.0, 0.5, 1.0])
    r["half_life_min_median_max"] = [float(x) for x in q]
    r["error_min_median_max"] = [float(x) for x in np.quantile(er, [0.0, 0.5, 1.0])]
    print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
