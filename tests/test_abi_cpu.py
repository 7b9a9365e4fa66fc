"""The C-ABI library on a machine without a GPU: it loads, exports every entry point
include/stq.h declares, computes pool layouts that agree with the oracle's own layout,
and rejects bad descriptions with the documented status codes."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import stq_oracle as O
from quantized_linear_attention_02_b200 import build, stq
from quantized_linear_attention_02_b200 import workload as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return stq.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "stq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(stq_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    # and nothing else in the header is left without a definition
    assert "stq_decode_step" in names and "stq_quantize_init" in names


def test_version(lib):
    assert b"sm_100a" in lib.stq_version()


@pytest.mark.parametrize("w", W.WORKLOADS, ids=lambda w: w.name)
def test_layout_matches_oracle_layout(lib, w):
    ub, rb = W.unit_bits(w), W.row_bits(w)
    om = W.omega(w)
    n_slots = W.n_slots(w.B)
    got = stq.layout(w.kind, n_slots, ub, om)
    L = O.Layout(rb)
    assert got["slot_code_bytes"] == L.slot_code_bytes
    assert got["codes_bytes"] == n_slots * L.slot_code_bytes
    assert got["n_pivot_rows"] == L.n_pivot_rows
    assert got["scales_bytes"] == n_slots * w.H * 2 * 128 * 4
    assert got["pivots_bytes"] == n_slots * L.n_pivot_rows * 128 * 2
    heads = [int(L.code_len[h].sum() + 256 * (rb[h] == 16).sum()) for h in range(w.H)]
    assert got["max_head_bytes"] == max(heads)


@pytest.mark.parametrize("seed", range(12))
def test_layout_matches_oracle_layout_random_widths(lib, seed):
    # random width maps: either kind, 1..5 heads, every width, pivot-only heads
    rng = np.random.default_rng(500 + seed)
    kind = ("gdn", "kda")[seed % 2]
    H = int(rng.integers(1, 6))
    n_slots = int(rng.integers(1, 9))
    widths = np.array([2, 4, 6, 8, 16], np.uint8)
    if kind == "gdn":
        ub = rng.choice(widths, H)
        rb = np.repeat(ub[:, None], 128, 1)
    else:
        rb = rng.choice(widths, (H, 128), p=[0.2, 0.3, 0.2, 0.2, 0.1]).astype(np.uint8)
        if H > 1:
            rb[H - 1] = 16 if seed % 4 == 1 else rb[H - 1]      # an all-pivot head
        ub = rb.reshape(-1)
    om = rng.lognormal(0, 1, (H, 128)).astype(np.float32)
    got = stq.layout(kind, n_slots, ub.astype(np.uint8), om)
    L = O.Layout(rb)
    assert got["slot_code_bytes"] == L.slot_code_bytes
    assert got["codes_bytes"] == n_slots * L.slot_code_bytes
    assert got["n_pivot_rows"] == L.n_pivot_rows
    assert got["scales_bytes"] == n_slots * H * 2 * 128 * 4
    assert got["pivots_bytes"] == n_slots * L.n_pivot_rows * 128 * 2
    heads = [int(L.code_len[h].sum() + 256 * (rb[h] == 16).sum()) for h in range(H)]
    assert got["max_head_bytes"] == max(heads)


@pytest.mark.parametrize("w", W.WORKLOADS[1:3], ids=lambda w: w.name)
def test_absmax_scheme_keeps_the_layout(lib, w):
    args = (w.kind, W.n_slots(w.B), W.unit_bits(w), W.omega(w))
    assert stq.layout(*args, "row_absmax") == stq.layout(*args)


@pytest.mark.parametrize("w", W.WORKLOADS[1:3], ids=lambda w: w.name)
def test_binary16_scales_halve_the_scale_bytes(lib, w):
    args = (w.kind, W.n_slots(w.B), W.unit_bits(w), W.omega(w))
    a, b = stq.layout(*args), stq.layout(*args, "stepquant", 16)
    assert b["scales_bytes"] * 2 == a["scales_bytes"]
    assert {k: v for k, v in a.items() if k != "scales_bytes"} == {k: v for k, v in b.items() if k != "scales_bytes"}
    assert stq.layout(*args, "stepquant", 0) == a


def test_six_bit_head_size(lib):
    got = stq.layout("gdn", 1, np.array([6], np.uint8), np.ones((1, 128), np.float32))
    assert got["slot_code_bytes"] == 128 * 96        # 4 codes in 3 bytes


@pytest.mark.parametrize("bad", ["width", "omega_zero", "omega_nan", "kind", "slots", "scheme", "scale_bits"])
def test_invalid_descriptions_rejected(lib, bad):
    ub = np.full(4, 6, np.uint8)
    om = np.ones((4, 128), np.float32)
    kind, n_slots, scheme = "gdn", 3, "stepquant"
    if bad == "width":
        ub[2] = 5
    elif bad == "omega_zero":
        om[1, 7] = 0
    elif bad == "omega_nan":
        om[0, 0] = np.nan
    elif bad == "kind":
        kind = 7
    elif bad == "slots":
        n_slots = 0
    elif bad == "scheme":
        scheme = 2
    scale_bits = 8 if bad == "scale_bits" else 32
    with pytest.raises(stq.StqError) as e:
        stq.layout(kind, n_slots, ub, om, scheme, scale_bits)
    assert e.value.status == 1
    assert lib.stq_last_error()


def test_null_arguments(lib):
    assert lib.stq_pool_layout(None, None) == 1
    assert lib.stq_decode_step(None, None, 1, None, None, None, None, None, None, None) == 1
    assert lib.stq_pool_check(None, None) == 1
    lib.stq_pool_destroy(None)
    assert lib.stq_fp32_decode_step(3, 1, 1, 128, None, None, None, None, None, None, None, None) == 1
    assert lib.stq_fp32_decode_step(0, 1, 1, 64, None, None, None, None, None, None, None, None) == 1


def test_pipeline_and_in_head_error_reject_bad_arguments_without_a_gpu(lib):
    # argument checks come before any CUDA call, so they run here
    vp = ctypes.c_void_p
    assert lib.stq_pipeline_staging_bytes(None, 4) == 0
    out = vp(123)
    st = lib.stq_pipeline_create(None, 4, vp(16), ctypes.c_size_t(1 << 20), ctypes.byref(out))
    assert st == 1 and out.value is None and lib.stq_last_error()
    st = lib.stq_pipeline_step(None, vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), None)
    assert st == 1 and b"pipeline" in lib.stq_last_error()
    assert lib.stq_pipeline_finish(None, None) == 1
    lib.stq_pipeline_destroy(None)                       # NULL is ignored
    cand = (ctypes.c_int * 1)(6)
    st = lib.stq_row_error_at_widths(None, vp(16), 1, vp(16), ctypes.cast(cand, vp), 1, vp(16), None)
    assert st == 1 and b"pool" in lib.stq_last_error()


def test_issue_rate_probe_rejects_bad_arguments_without_a_gpu(lib):
    vp = ctypes.c_void_p
    assert lib.stq_issue_rate_probe(3, 1, 1, vp(16), None) == 1
    assert b"mode" in lib.stq_last_error()
    assert lib.stq_issue_rate_probe(0, 0, 1, vp(16), None) == 1
    assert lib.stq_issue_rate_probe(0, 65536, 1, vp(16), None) == 1
    assert lib.stq_issue_rate_probe(1, 1, 0, vp(16), None) == 1
    assert lib.stq_issue_rate_probe(2, 1, 1, None, None) == 1
    assert b"d_out" in lib.stq_last_error()
