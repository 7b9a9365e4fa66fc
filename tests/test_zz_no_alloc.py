"""stq_decode_step_host_static: the host-buffer decode step for callers that cannot
allocate device memory on their decode path (its device staging is a fixed array the
library declares). It must give the results of stq_decode_step_host, whose staging the
caller allocates, call after call. This file runs last so that a failure here comes
after every other test has run."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from quantized_linear_attention_02_b200 import build, stq  # noqa: E402
from quantized_linear_attention_02_b200 import workload as W  # noqa: E402

import stq_testlib as T  # noqa: E402

D = 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    build.build()
    stq.lib()


def _snapshot(pool):
    return pool.codes.clone(), pool.scales.clone(), pool.pivots.clone()


def _restore(pool, snap):
    pool.codes.copy_(snap[0])
    pool.scales.copy_(snap[1])
    pool.pivots.copy_(snap[2])


@pytest.mark.parametrize("widx", [1, 2])
def test_static_staging_matches_caller_staging(widx):
    w = W.WORKLOADS[widx]
    reqs = [0, 1, 2, 3]
    pool = stq.Pool(w.kind, W.n_slots(w.B), W.unit_bits(w), W.omega(w))
    slots = torch.tensor([W.slot_of_request(b) for b in reqs], dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    S0 = torch.randn((len(reqs), w.H, D, D), device="cuda", generator=g) * 0.1
    pool.quantize_init(slots, S0)
    pool.check()
    start = _snapshot(pool)
    steps = [T.inputs_for(w, "decode", t, reqs) for t in range(2)]
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()

    # the existing entry point, with a staging buffer the caller allocates
    staging = torch.empty(pool.host_staging_bytes(len(reqs)), dtype=torch.uint8, device="cuda")
    ref_out, ref_state = [], []
    for x in steps:
        h_out = torch.empty((len(reqs), w.H, D)).pin_memory()
        pool.decode_step_host(slots, pin(x.q), pin(x.k), pin(x.v), pin(x.gate), pin(x.beta), h_out, staging)
        torch.cuda.synchronize()
        ref_out.append(h_out.clone())
        ref_state.append(_snapshot(pool))
    pool.check()

    # the static-staging entry point, two calls in a row from the same start
    _restore(pool, start)
    for t, x in enumerate(steps):
        h_out = torch.empty((len(reqs), w.H, D)).pin_memory()
        pool.decode_step_host_static(slots, pin(x.q), pin(x.k), pin(x.v), pin(x.gate), pin(x.beta), h_out)
        torch.cuda.synchronize()
        assert torch.equal(h_out, ref_out[t]), f"readout differs after call {t}"
        assert torch.equal(pool.codes, ref_state[t][0]), f"codes differ after call {t}"
        assert torch.equal(pool.scales, ref_state[t][1]), f"scales differ after call {t}"
        assert torch.equal(pool.pivots, ref_state[t][2]), f"pivots differ after call {t}"
    pool.check()


def test_static_staging_at_its_largest_batch():
    """GDN with 48 heads: 85 requests (4,080 head-states) is the largest batch whose
    staging fits the static array; it must match the caller-staged entry point."""
    w = W.WORKLOADS[1]
    B = 85
    pool = stq.Pool(w.kind, W.n_slots(B), W.unit_bits(w), W.omega(w))
    assert pool.host_staging_bytes(B) <= stq.STATIC_STAGING_BYTES < pool.host_staging_bytes(B + 1)
    slots = torch.tensor([W.slot_of_request(b) for b in range(B)], dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    pool.quantize_init(slots, torch.randn((B, w.H, D, D), device="cuda", generator=g) * 0.1)
    pool.check()
    start = _snapshot(pool)
    gen = torch.Generator(device="cuda").manual_seed(12)
    x = [t.cpu().pin_memory() for t in W.torch_step_inputs(w, B, gen, "cuda")]
    staging = torch.empty(pool.host_staging_bytes(B), dtype=torch.uint8, device="cuda")
    ref = torch.empty((B, w.H, D)).pin_memory()
    pool.decode_step_host(slots, *x, ref, staging)
    torch.cuda.synchronize()
    after = _snapshot(pool)
    _restore(pool, start)
    got = torch.full((B, w.H, D), float("nan")).pin_memory()
    pool.decode_step_host_static(slots, *x, got)
    torch.cuda.synchronize()
    pool.check()
    assert torch.equal(got, ref)
    assert all(torch.equal(a, b) for a, b in zip(_snapshot(pool), after))


def test_static_staging_rejects_a_batch_beyond_its_size():
    w = W.WORKLOADS[3]
    pool = stq.Pool(w.kind, 4, W.unit_bits(w), W.omega(w))
    B = 512                                  # 512 x 48 head-states need ~50 MB of staging
    slots = torch.zeros(B, dtype=torch.int32, device="cuda")
    h = torch.zeros((B, w.H, D))
    hg = torch.zeros((B, w.H))
    with pytest.raises(stq.StqError) as e:
        pool.decode_step_host_static(slots, h, h, h, hg, hg, h)
    assert e.value.status == 1
    assert "static" in str(e.value)
