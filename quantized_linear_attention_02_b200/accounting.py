"""Memory accounting of a packed state pool against its FP32 form.

The pages compare a packed state pool with the FP32 one by compression ratio, bits per
stored state value and pool totals: the singularity-lens summary, numbers paragraph
(state compression, compact bits per value including scales and FP16 pivots), and the
zhichai.net forum reply, which recomputes the pool sizes from the slot count and the
per-slot bytes (the 2,304 Qwen heads are named in the bloombook.cn tutorial, section
three).
This module does that arithmetic for the library's own layout: the packed bytes per slot
come from stq_pool_layout (codes, row and column scales, FP16 pivot rows), never from a
separate formula.

Definitions (one head-state has d_k * d_v = 128 * 128 values, 4 bytes each in FP32):
  compression     = FP32 state bytes / packed state bytes
  bits per value  = 8 * packed state bytes / number of state values
  pool totals     = n_slots * (state bytes + other per-slot bytes), in GiB (2^30 bytes)
Host only: no CUDA call.
"""
from __future__ import annotations

import argparse
import json

import numpy as np

from . import stq
from . import workload as W

D = 128
VALUES_PER_HEAD = D * D
FP32_HEAD_BYTES = 4 * VALUES_PER_HEAD
MiB = float(1 << 20)
GiB = float(1 << 30)


def state_accounting(packed_state_bytes: float, n_heads: int) -> dict:
    """Compression and bits per value of n_heads head-states held in packed_state_bytes."""
    fp32 = float(n_heads * FP32_HEAD_BYTES)
    return {
        "fp32_bytes": fp32,
        "packed_bytes": float(packed_state_bytes),
        "compression": fp32 / float(packed_state_bytes),
        "bits_per_value": 8.0 * float(packed_state_bytes) / float(n_heads * VALUES_PER_HEAD),
    }


def pool_totals(fp32_state_bytes: float, packed_state_bytes: float, other_bytes: float, n_slots: int) -> dict:
    """Pool sizes in GiB for n_slots slots, each holding its state plus other_bytes."""
    fp32 = n_slots * (fp32_state_bytes + other_bytes) / GiB
    packed = n_slots * (packed_state_bytes + other_bytes) / GiB
    return {"fp32_gib": fp32, "packed_gib": packed, "saved_gib": fp32 - packed}


def slot_state_bytes(kind, unit_bits, omega, scale_bits: int = 32) -> int:
    """Packed bytes of one slot of a pool with these widths: codes + scales + pivot rows,
    as the library lays them out."""
    s = stq.layout(kind, 1, np.asarray(unit_bits, np.uint8), np.asarray(omega, np.float32),
                   "stepquant", scale_bits)
    return int(s["codes_bytes"] + s["scales_bytes"] + s["pivots_bytes"])


def workload_accounting(w, scale_bits: int = 32, model_heads: int | None = None,
                        n_slots: int | None = None, other_bytes: float = 0.0) -> dict:
    """Accounting of a workload's allocation; with model_heads, its per-head average is
    carried over to a model of that many heads (and n_slots slots of it)."""
    packed = slot_state_bytes(w.kind, W.unit_bits(w), W.omega(w), scale_bits)
    out = {"workload": w.name, "scale_bits": scale_bits, "heads": w.H,
           **state_accounting(packed, w.H)}
    if model_heads is not None:
        per_head = packed / w.H
        out["model_heads"] = model_heads
        out["model_packed_mib"] = per_head * model_heads / MiB
        out["model_fp32_mib"] = model_heads * FP32_HEAD_BYTES / MiB
        if n_slots is not None:
            out.update(pool_totals(model_heads * FP32_HEAD_BYTES, per_head * model_heads,
                                   other_bytes, n_slots))
            out["n_slots"] = n_slots
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description="memory accounting of a packed state pool")
    ap.add_argument("--workload", type=int, default=3, help="index into the workload list")
    ap.add_argument("--scale-bits", type=int, choices=[32, 16], default=32)
    ap.add_argument("--model-heads", type=int, default=None, help="carry the per-head bytes to this many heads")
    ap.add_argument("--slots", type=int, default=None, help="slots of the pool (with --model-heads)")
    ap.add_argument("--other-mib", type=float, default=0.0, help="non-state MiB per slot (with --slots)")
    a = ap.parse_args(argv)
    print(json.dumps(workload_accounting(W.WORKLOADS[a.workload], a.scale_bits, a.model_heads,
                                         a.slots, a.other_mib * MiB)))


if __name__ == "__main__":
    main()
