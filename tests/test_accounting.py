"""Memory accounting helper: its arithmetic reproduces the pages' own figures from the
pages' inputs, and on the library's layout it gives the closed-form bytes of simple pools
and the oracle layout's bytes of the workload allocations."""
import numpy as np
import pytest

from oracle import stq_oracle as O
from quantized_linear_attention_02_b200 import accounting as A
from quantized_linear_attention_02_b200 import build
from quantized_linear_attention_02_b200 import workload as W

MiB = 1 << 20


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def test_pages_memory_figures():
    # zhichai.net forum reply and singularity-lens numbers paragraph: 2,304 Qwen heads
    # of 64 KiB FP32 state = 144 MiB per slot; 28.625 MiB packed at nominal 6 bits;
    # 2.8125 MiB of other per-slot state; (5 * 512 + 1) slots
    st = A.state_accounting(28.625 * MiB, 2304)
    assert st["fp32_bytes"] == 144 * MiB
    assert round(st["compression"], 4) == 5.0306
    assert round(st["bits_per_value"], 3) == 6.361
    tot = A.pool_totals(144 * MiB, 28.625 * MiB, 2.8125 * MiB, 5 * 512 + 1)
    assert round(tot["fp32_gib"], 2) == 367.17
    assert round(tot["packed_gib"], 2) == 78.62
    assert round(tot["saved_gib"], 2) == 288.55


@pytest.mark.parametrize("bits,scale_bits,expect", [
    (8, 32, 8.5), (6, 32, 6.5), (4, 32, 4.5), (2, 32, 2.5), (16, 32, 16.5),
    (8, 16, 8.25), (6, 16, 6.25), (2, 16, 2.25),
])
def test_uniform_head_bits_per_value(bits, scale_bits, expect):
    # one head of width b: 128 rows of 16 b bytes (or 128 FP16 rows) plus r[128], c[128]
    st = A.state_accounting(A.slot_state_bytes("gdn", [bits], np.ones((1, 128), np.float32), scale_bits), 1)
    assert st["bits_per_value"] == expect


@pytest.mark.parametrize("w", W.WORKLOADS, ids=lambda w: w.name)
@pytest.mark.parametrize("scale_bits", [32, 16])
def test_workload_bytes_match_oracle_layout(w, scale_bits):
    L = O.Layout(W.row_bits(w))
    expect = L.slot_code_bytes + L.n_pivot_rows * 128 * 2 + w.H * 2 * 128 * scale_bits // 8
    got = A.workload_accounting(w, scale_bits)
    assert got["packed_bytes"] == expect
    assert got["bits_per_value"] == 8.0 * expect / (w.H * 128 * 128)


def test_throughput_workload_at_model_scale():
    # the nominal 6-bit GDN allocation of the throughput workload carried to 2,304 heads
    # and the pages' slot count: smaller than FP32 by the per-head compression
    w = W.WORKLOADS[3]
    got = A.workload_accounting(w, 32, model_heads=2304, n_slots=5 * 512 + 1, other_bytes=2.8125 * MiB)
    assert got["model_fp32_mib"] == 144.0
    assert abs(got["model_fp32_mib"] / got["model_packed_mib"] - got["compression"]) < 1e-12
    assert round(got["fp32_gib"], 2) == 367.17
    assert got["packed_gib"] < got["fp32_gib"] / 4
