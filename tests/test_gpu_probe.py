"""The issue-rate probe that the bench times for the measured peak of its ALU roofline:
it runs in every mode, its integer mode computes what it states (checked exactly on the
CPU), and the lane-operation count it reports follows its launch."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from quantized_linear_attention_02_b200 import build, stq  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    build.build()
    stq.lib()


def _lop3_expected(blocks, iters):
    # lop3 with table 0x96 is a ^ b ^ c: each chain toggles by y ^ z once per iteration
    T = stq.PROBE_THREADS
    out = np.empty(blocks * T, np.float32)
    for b in range(blocks):
        for t in range(T):
            y = (0x9E3779B9 ^ t) & 0xFFFFFFFF
            z = (0x7F4A7C15 + b) & 0xFFFFFFFF
            x = 0
            for i in range(8):
                a = (t * 2654435761 + i) & 0xFFFFFFFF
                if iters & 1:
                    a ^= y ^ z
                x ^= a
            out[b * T + t] = np.float32(x & 0xFFFF)
    return out


@pytest.mark.parametrize("iters", [1, 6, 7])
def test_integer_mode_matches_its_definition(iters):
    blocks = 3
    out = torch.empty(blocks * stq.PROBE_THREADS, device="cuda")
    ops = stq.issue_rate_probe(2, blocks, iters, out)
    torch.cuda.synchronize()
    assert ops == blocks * stq.PROBE_THREADS * 8 * iters
    assert np.array_equal(out.cpu().numpy(), _lop3_expected(blocks, iters))


@pytest.mark.parametrize("mode", [0, 1])
def test_float_modes_run_and_repeat(mode):
    blocks, iters = 2, 1000
    a = torch.empty(blocks * stq.PROBE_THREADS, device="cuda")
    b = torch.empty_like(a)
    ops = stq.issue_rate_probe(mode, blocks, iters, a)
    stq.issue_rate_probe(mode, blocks, iters, b)
    torch.cuda.synchronize()
    assert ops == blocks * stq.PROBE_THREADS * 8 * iters * (2 if mode == 0 else 1)
    assert torch.isfinite(a).all() and torch.equal(a, b)


def test_bench_issue_rates_are_positive():
    import bench
    rates = bench.issue_rates(torch.cuda.current_stream(), reps=1)
    assert rates["ffma2"] > 0 and rates["lop3"] > 0
