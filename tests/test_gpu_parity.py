"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on the five
workloads. Every expected value comes from the oracle on the same seeded inputs;
the initial states the GPU receives are oracle-built too."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from oracle import stq_oracle as O  # noqa: E402
from quantized_linear_attention_02_b200 import build, stq  # noqa: E402
from quantized_linear_attention_02_b200 import workload as W  # noqa: E402

import stq_testlib as T  # noqa: E402

D = 128
F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    build.build()
    stq.lib()


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def slots_t(reqs):
    return dev(np.array([W.slot_of_request(b) for b in reqs], np.int32))


def make_pool(w, n_slots=None):
    ub = W.unit_bits(w)
    om = W.omega(w)
    return stq.Pool(w.kind, n_slots or W.n_slots(w.B), ub, om), O.Layout(W.row_bits(w)), om


def oracle_quantised(w, reqs):
    S0 = T.warm_state(w.index, tuple(reqs))
    u, r, c, piv = O.refit(S0, W.omega(w), W.row_bits(w))
    return S0, u, r, c, piv


# ---------------------------------------------------------------------------------
# FP32 step
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("widx", [0, 2])
def test_fp32_step_bit_exact_state(widx):
    w = W.WORKLOADS[widx]
    reqs = list(range(min(w.B, 2)))
    S0 = T.warm_state(widx, tuple(reqs), steps=8)
    x = T.inputs_for(w, "decode", 0, reqs)
    S_or, o_or = O.fp32_step(S0, x.q, x.k, x.v, O.gate_rows(x.gate, w.kind, D), x.beta)
    S = dev(S0)
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    stq.fp32_decode_step(w.kind, S, dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
    torch.cuda.synchronize()
    assert np.array_equal(S.cpu().numpy(), S_or)
    assert T.per_vector_rel_l2(out.cpu().numpy(), o_or).max() <= T.OUT_REL_L2


# ---------------------------------------------------------------------------------
# dequantise / quantise
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("widx", [0, 1, 2])
def test_dequantize_bit_exact(widx):
    w = W.WORKLOADS[widx]
    reqs = [0, min(3, w.B - 1)] if w.B > 1 else [0]
    pool, L, _ = make_pool(w)
    S0, u, r, c, piv = oracle_quantised(w, reqs)
    slots = [W.slot_of_request(b) for b in reqs]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    out = torch.empty((len(reqs), w.H, D, D), device="cuda")
    pool.dequantize(slots_t(reqs), out)
    pool.check()
    assert np.array_equal(out.cpu().numpy(), O.dequantize(u, r, c, piv, W.row_bits(w)))


@pytest.mark.parametrize("widx", [0, 1, 2])
def test_quantize_init_matches_oracle(widx):
    w = W.WORKLOADS[widx]
    reqs = [0, min(5, w.B - 1)] if w.B > 1 else [0]
    pool, L, _ = make_pool(w)
    S0, u, r, c, piv = oracle_quantised(w, reqs)
    pool.quantize_init(slots_t(reqs), dev(S0))
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, [W.slot_of_request(b) for b in reqs])
    rb = W.row_bits(w)
    n = T.compare_codes(ug, u, S0, r, c, rb, "quantize_init", config=w.name)
    T.check_scales(rg, r, cg, c, n, "quantize_init")
    piv_rows = (rb == 16)
    assert np.array_equal(pg[:, piv_rows], piv[:, piv_rows])


# ---------------------------------------------------------------------------------
# decode step, teacher-forced from an identical packed state
# ---------------------------------------------------------------------------------
def _single_step(w, reqs, t, pool, L):
    S0, u, r, c, piv = oracle_quantised(w, reqs)
    slots = [W.slot_of_request(b) for b in reqs]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    x = T.inputs_for(w, "decode", t, reqs)
    rb = W.row_bits(w)
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, rb, W.omega(w), x.q, x.k, x.v,
                                         O.gate_rows(x.gate, w.kind, D), x.beta)
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    pool.decode_step(slots_t(reqs), dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u2, X, r2, c2, rb, f"{w.name} step {t}", config=w.name)
    T.check_scales(rg, r2, cg, c2, n, f"{w.name} step {t}")
    piv_rows = rb == 16
    assert np.array_equal(pg[:, piv_rows], p2[:, piv_rows])
    assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2
    return n


@pytest.mark.parametrize("widx,t", [(0, 0), (0, 7), (1, 0), (1, 31), (2, 0), (2, 17)])
def test_decode_step_teacher_forced(widx, t):
    w = W.WORKLOADS[widx]
    reqs = [0, w.B - 1] if w.B > 1 else [0]
    pool, L, _ = make_pool(w)
    _single_step(w, reqs, t, pool, L)


# ---------------------------------------------------------------------------------
# chained steps: each side runs on its own from the same start
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("widx,steps", [(0, 16), (1, 64), (2, 64)])
def test_decode_chain(widx, steps):
    w = W.WORKLOADS[widx]
    reqs = [1, w.B - 2] if w.B > 2 else [0]
    pool, L, _ = make_pool(w)
    S0, u, r, c, piv = oracle_quantised(w, reqs)
    slots = [W.slot_of_request(b) for b in reqs]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    rb, om = W.row_bits(w), W.omega(w)
    st = slots_t(reqs)
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    worst_o = 0.0
    for t in range(steps):
        x = T.inputs_for(w, "decode", t, reqs)
        u, r, c, piv, o, X = O.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v,
                                           O.gate_rows(x.gate, w.kind, D), x.beta)
        pool.decode_step(st, dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
        worst_o = max(worst_o, T.per_vector_rel_l2(out.cpu().numpy(), o).max())
    pool.check()
    Sg = torch.empty((len(reqs), w.H, D, D), device="cuda")
    pool.dequantize(st, Sg)
    S_or = O.dequantize(u, r, c, piv, rb)
    assert T.rel_l2(Sg.cpu().numpy(), S_or) <= T.CHAIN_REL_L2
    assert worst_o <= T.OUT_REL_L2


# ---------------------------------------------------------------------------------
# full-size workloads in the launch configuration the bench times
# ---------------------------------------------------------------------------------
def _full_size_start(w, pool, L, sample):
    """Quantise every request's state (random ones, oracle-built warm states for the
    sampled requests) and check the sample against the oracle's quantiser; then put the
    oracle's packed state into the sampled slots so that later steps start identical.
    Returns the oracle's packed state of the sample."""
    om, rb = W.omega(w), W.row_bits(w)
    g = torch.Generator(device="cuda").manual_seed(1234 + w.index)
    S_all = torch.randn((w.B, w.H, D, D), device="cuda", generator=g) * 0.05
    S0 = T.warm_states(w.index, sample)
    S_all[sample] = dev(S0)
    pool.quantize_init(slots_t(range(w.B)), S_all)
    del S_all
    pool.check()
    u, r, c, piv = O.refit(S0, om, rb)
    slots = [W.slot_of_request(b) for b in sample]
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u, S0, r, c, rb, "full-size quantize_init", config=w.name)
    T.check_scales(rg, r, cg, c, n, "full-size quantize_init")
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    return u, r, c, piv


def _full_size_inputs(w, t, sample, gen):
    """Inputs of step t for all B requests: the recipe's distributions from the device
    RNG, with the sampled requests' inputs from their seeded NumPy streams."""
    xin = dict(zip(("q", "k", "v", "gate", "beta"), W.torch_step_inputs(w, w.B, gen, "cuda")))
    xs = T.inputs_for(w, "decode", t, sample)
    for name in xin:
        xin[name][sample] = dev(getattr(xs, name))
    return xin, xs


@pytest.mark.parametrize("widx", [3, 4])
def test_full_size_sampled(widx):
    w = W.WORKLOADS[widx]
    pool, L, om = make_pool(w)
    sample = [int(b) for b in W.parity_sample(w, 8)]
    u, r, c, piv = _full_size_start(w, pool, L, sample)
    gen = torch.Generator(device="cuda").manual_seed(99)
    xin, xs = _full_size_inputs(w, 0, sample, gen)
    out = torch.empty((w.B, w.H, D), device="cuda")
    pool.decode_step(slots_t(range(w.B)), xin["q"], xin["k"], xin["v"], xin["gate"], xin["beta"], out)
    pool.check()
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, W.row_bits(w), om, xs.q, xs.k, xs.v,
                                         O.gate_rows(xs.gate, w.kind, D), xs.beta)
    ug, rg, cg, pg = T.read_pool_state(pool, L, [W.slot_of_request(b) for b in sample])
    n = T.compare_codes(ug, u2, X, r2, c2, W.row_bits(w), "full-size decode", config=w.name)
    T.check_scales(rg, r2, cg, c2, n, "full-size decode")
    assert T.per_vector_rel_l2(out[sample].cpu().numpy(), o).max() <= T.OUT_REL_L2
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("widx", [3, 4])
def test_full_size_chained(widx):
    """64 chained steps of the full-B launch; the 8 sampled requests run on their own
    on both sides from one packed start: every step's readout and the final
    dequantised states are compared with the oracle's chains."""
    w = W.WORKLOADS[widx]
    steps = 64
    pool, L, om = make_pool(w)
    rb = W.row_bits(w)
    sample = [int(b) for b in W.parity_sample(w, 8)]
    start = _full_size_start(w, pool, L, sample)
    chains = T.oracle_chains(widx, sample, start, 0, steps)
    gen = torch.Generator(device="cuda").manual_seed(199 + widx)
    all_slots = slots_t(range(w.B))
    out = torch.empty((w.B, w.H, D), device="cuda")
    worst_o = 0.0
    for t in range(steps):
        xin, _ = _full_size_inputs(w, t, sample, gen)
        pool.decode_step(all_slots, xin["q"], xin["k"], xin["v"], xin["gate"], xin["beta"], out)
        o_or = np.stack([ch[0][t] for ch in chains])
        worst_o = max(worst_o, T.per_vector_rel_l2(out[sample].cpu().numpy(), o_or).max())
    pool.check()
    assert torch.isfinite(out).all()
    Sg = torch.empty((len(sample), w.H, D, D), device="cuda")
    pool.dequantize(slots_t(sample), Sg)
    fin = [ch[1] for ch in chains]
    S_or = np.concatenate([O.dequantize(*st, rb) for st in fin], 0)
    rel = T.rel_l2(Sg.cpu().numpy(), S_or)
    ug = T.read_pool_state(pool, L, [W.slot_of_request(b) for b in sample])[0]
    u_or = np.concatenate([st[0] for st in fin], 0)
    quant = np.broadcast_to((rb != 16)[..., None], u_or.shape)
    T.REPORTS[f"{w.name} 64 chained steps, 8 sampled requests"] = (
        f"state rel L2 {rel:.3g}, worst readout rel L2 {worst_o:.3g}, "
        f"final codes differing {int(((ug != u_or) & quant).sum())} of {int(quant.sum())}")
    assert rel <= T.CHAIN_REL_L2
    assert worst_o <= T.OUT_REL_L2


# ---------------------------------------------------------------------------------
# edge cases and error paths
# ---------------------------------------------------------------------------------
def test_bad_slot_is_flagged_and_skipped():
    w = W.WORKLOADS[0]
    pool, L, _ = make_pool(w, n_slots=3)
    S = torch.zeros((2, w.H, D, D), device="cuda")
    pool.quantize_init(dev(np.array([0, 2], np.int32)), S)
    pool.check()
    before = pool.codes.clone()
    x = W.step_inputs(w, "decode", 0, 0, 1)
    out = torch.zeros((2, w.H, D), device="cuda")
    rep = lambda a: dev(np.concatenate([a, a]))
    pool.decode_step(dev(np.array([1, 7], np.int32)), rep(x.q), rep(x.k), rep(x.v), rep(x.gate),
                     rep(x.beta), out)
    with pytest.raises(stq.StqError) as e:
        pool.check()
    assert e.value.status == 4
    pool.check()            # the error bit was cleared
    sz = pool.sizes["slot_code_bytes"]
    assert torch.equal(pool.codes[:sz], before[:sz])           # slot 0 untouched
    assert torch.count_nonzero(out[1]) == 0                    # skipped request


@pytest.mark.parametrize("kind,ub,B", [("gdn", (6,), 1), ("gdn", (2, 16, 8), 5), ("kda", 5, 3), ("kda", 7, 41)])
def test_odd_item_counts(kind, ub, B):
    """Batches whose (request, head) count is odd or smaller than the grid: each CTA of
    the decode kernel runs two groups on alternate items, so the second group of the
    last CTA may get none. Two teacher-forced steps on odd slot indices."""
    rng = np.random.default_rng(B)
    if kind == "gdn":
        ub = np.array(ub, np.uint8)
        H = ub.size
        rb = np.repeat(ub[:, None], D, axis=1)
    else:
        H = ub
        rb = rng.choice([2, 4, 6, 8, 16], size=(H, D), p=[0.2, 0.3, 0.2, 0.25, 0.05])
        ub = rb.reshape(-1).astype(np.uint8)
    om = rng.lognormal(0, 1, (H, D)).astype(F32)
    pool = stq.Pool(kind, 2 * B + 1, ub, om)
    L = O.Layout(rb)
    slots = [2 * b + 1 for b in range(B)]
    st = dev(np.array(slots, np.int32))
    S0 = (rng.standard_normal((B, H, D, D)) * rng.lognormal(0, 1, (B, H, D, 1)) * 0.1).astype(F32)
    u, r, c, piv = O.refit(S0, om, rb)
    out = torch.empty((B, H, D), device="cuda")
    for t in range(2):
        q = rng.standard_normal((B, H, D))
        k = rng.standard_normal((B, H, D))
        q = (q / np.linalg.norm(q, axis=-1, keepdims=True)).astype(F32)
        k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(F32)
        v = rng.standard_normal((B, H, D)).astype(F32)
        gate = np.exp(rng.uniform(-0.2, -0.001, (B, H) if kind == "gdn" else (B, H, D))).astype(F32)
        beta = (1 / (1 + np.exp(-rng.standard_normal((B, H))))).astype(F32)
        T.write_oracle_state(pool, L, slots, u, r, c, piv)
        u, r, c, piv, o, X = O.decode_step(u, r, c, piv, rb, om, q, k, v, O.gate_rows(gate, kind, D), beta)
        pool.decode_step(st, dev(q), dev(k), dev(v), dev(gate), dev(beta), out)
        pool.check()
        ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
        what = f"{kind} H={H} B={B} step {t}"
        n = T.compare_codes(ug, u, X, r, c, rb, what, config=f"{kind} odd item counts")
        T.check_scales(rg, r, cg, c, n, what)
        assert np.array_equal(pg[:, rb == 16], piv[:, rb == 16])
        assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2


def test_empty_batch_is_a_no_op():
    w = W.WORKLOADS[0]
    pool, L, _ = make_pool(w, n_slots=2)
    e = torch.empty(0, device="cuda")
    pool.decode_step(torch.empty(0, dtype=torch.int32, device="cuda"), e, e, e, e, e, e)
    pool.check()


def test_zero_state_stays_zero_and_all_pivot_kda_head():
    # a KDA head whose rows are all FP16 pivots, next to a zero state
    ub = np.full(2 * D, 6, np.uint8)
    ub[D:] = 16
    om = np.ones((2, D), F32)
    rb = ub.reshape(2, D)
    pool = stq.Pool("kda", 2, ub, om)
    L = O.Layout(rb)
    rng = np.random.default_rng(0)
    S0 = np.zeros((1, 2, D, D), F32)
    S0[0, 1] = rng.standard_normal((D, D)).astype(F32)
    st = dev(np.array([1], np.int32))
    pool.quantize_init(st, dev(S0))
    u, r, c, piv = O.refit(S0, om, rb)
    ug, rg, cg, pg = T.read_pool_state(pool, L, [1])
    assert np.array_equal(ug, u) and np.array_equal(rg, r) and np.array_equal(cg, c)
    assert np.array_equal(pg[:, rb == 16], piv[:, rb == 16])
    q = rng.standard_normal((1, 2, D)).astype(F32)
    k = (q / np.linalg.norm(q, axis=-1, keepdims=True)).astype(F32)
    v = rng.standard_normal((1, 2, D)).astype(F32)
    gate = np.full((1, 2, D), 0.9, F32)
    beta = np.full((1, 2), 0.5, F32)
    out = torch.empty((1, 2, D), device="cuda")
    pool.decode_step(st, dev(k), dev(k), dev(v), dev(gate), dev(beta), out)
    pool.check()
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, rb, om, k, k, v, gate, beta)
    ug, rg, cg, pg = T.read_pool_state(pool, L, [1])
    n = T.compare_codes(ug, u2, X, r2, c2, rb, "pivot head", config="kda_all_pivot_head")
    T.check_scales(rg, r2, cg, c2, n, "pivot head")
    assert np.array_equal(pg[:, rb == 16], p2[:, rb == 16])
    assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2


def test_host_entry_point_matches_device_entry_point():
    w = W.WORKLOADS[1]
    reqs = [0, 1, 2]
    pool, L, _ = make_pool(w)
    S0, u, r, c, piv = oracle_quantised(w, reqs)
    slots = [W.slot_of_request(b) for b in reqs]
    x = T.inputs_for(w, "decode", 3, reqs)
    out_dev = torch.empty((len(reqs), w.H, D), device="cuda")
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    pool.decode_step(slots_t(reqs), dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out_dev)
    pool.check()
    codes_dev = pool.codes.clone()
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    h_out = torch.empty((len(reqs), w.H, D)).pin_memory()
    staging = torch.empty(pool.host_staging_bytes(len(reqs)), dtype=torch.uint8, device="cuda")
    pool.decode_step_host(slots_t(reqs), pin(x.q), pin(x.k), pin(x.v), pin(x.gate), pin(x.beta),
                          h_out, staging)
    pool.check()
    assert torch.equal(pool.codes, codes_dev)
    assert torch.equal(h_out, out_dev.cpu())


@pytest.mark.parametrize("widx", [1, 2])
def test_pipelined_host_steps_match_serial_host_steps(widx):
    """The pipelined host-buffer steps (copies overlapping the neighbouring steps inside
    the library) give bit for bit the readouts and states of stq_decode_step_host."""
    w = W.WORKLOADS[widx]
    reqs = [0, 1, 2, 3, 4]
    steps = 4
    pool, L, _ = make_pool(w)
    S0, u, r, c, piv = oracle_quantised(w, reqs)
    slots = [W.slot_of_request(b) for b in reqs]
    st = slots_t(reqs)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    xs = [[pin(getattr(T.inputs_for(w, "decode", t, reqs), n)) for n in ("q", "k", "v", "gate", "beta")]
          for t in range(steps)]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    staging = torch.empty(pool.host_staging_bytes(len(reqs)), dtype=torch.uint8, device="cuda")
    ref = []
    for x in xs:
        h_out = torch.empty((len(reqs), w.H, D)).pin_memory()
        pool.decode_step_host(st, *x, h_out, staging)
        torch.cuda.synchronize()
        ref.append(h_out)
    pool.check()
    codes_ref, scales_ref = pool.codes.clone(), pool.scales.clone()
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    pipe = pool.pipeline(len(reqs))
    outs = [torch.full((len(reqs), w.H, D), float("nan")).pin_memory() for _ in range(steps)]
    for t, x in enumerate(xs):
        pipe.step(st, *x, outs[t])
        if t >= 1:      # on return the previous step's readout is on the host
            assert torch.equal(outs[t - 1], ref[t - 1]), f"step {t - 1}"
    pipe.finish()
    assert torch.equal(outs[-1], ref[-1])
    pipe.close()
    pool.check()
    assert torch.equal(pool.codes, codes_ref) and torch.equal(pool.scales, scales_ref)


# ---------------------------------------------------------------------------------
# the uniform baseline scheme: symmetric per-key-row absmax (same kernels, other
# quantiser)
# ---------------------------------------------------------------------------------
def make_absmax_pool(w, bits=None):
    ub = W.unit_bits(w) if bits is None else np.full_like(W.unit_bits(w), bits)
    rb = W.row_bits(w) if bits is None else np.full((w.H, D), bits)
    return stq.Pool(w.kind, W.n_slots(w.B), ub, W.omega(w), scheme="row_absmax"), O.Layout(rb), rb


@pytest.mark.parametrize("widx,bits", [(1, None), (2, None), (1, 6), (2, 4)])
def test_absmax_quantize_init_matches_oracle(widx, bits):
    w = W.WORKLOADS[widx]
    reqs = [0, w.B - 1]
    pool, L, rb = make_absmax_pool(w, bits)
    S0 = T.warm_state(w.index, tuple(reqs))
    u, r, c, piv = O.absmax_quantise(S0, rb)
    pool.quantize_init(slots_t(reqs), dev(S0))
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, [W.slot_of_request(b) for b in reqs])
    T.compare_codes(ug, u, S0, r, c, rb, "absmax quantize_init", config=f"{w.name} row_absmax")
    assert np.array_equal(rg, r) and np.array_equal(cg, c)
    assert np.array_equal(pg[:, rb == 16], piv[:, rb == 16])


@pytest.mark.parametrize("widx,t,bits", [(1, 0, None), (2, 5, None), (1, 3, 8), (2, 9, 2)])
def test_absmax_decode_step_teacher_forced(widx, t, bits):
    w = W.WORKLOADS[widx]
    reqs = [0, w.B - 1]
    pool, L, rb = make_absmax_pool(w, bits)
    S0 = T.warm_state(w.index, tuple(reqs))
    u, r, c, piv = O.absmax_quantise(S0, rb)
    slots = [W.slot_of_request(b) for b in reqs]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    x = T.inputs_for(w, "decode", t, reqs)
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, rb, W.omega(w), x.q, x.k, x.v,
                                         O.gate_rows(x.gate, w.kind, D), x.beta, scheme="row_absmax")
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    pool.decode_step(slots_t(reqs), dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    T.compare_codes(ug, u2, X, r2, c2, rb, f"absmax {w.name} step {t}", config=f"{w.name} row_absmax")
    assert np.array_equal(rg, r2) and np.array_equal(cg, c2)
    assert np.array_equal(pg[:, rb == 16], p2[:, rb == 16])
    assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2


@pytest.mark.parametrize("widx,steps", [(1, 16), (2, 16)])
def test_absmax_decode_chain(widx, steps):
    w = W.WORKLOADS[widx]
    reqs = [1, w.B - 2]
    pool, L, rb = make_absmax_pool(w)
    S0 = T.warm_state(w.index, tuple(reqs))
    u, r, c, piv = O.absmax_quantise(S0, rb)
    slots = [W.slot_of_request(b) for b in reqs]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    for t in range(steps):
        x = T.inputs_for(w, "decode", t, reqs)
        u, r, c, piv, o, _ = O.decode_step(u, r, c, piv, rb, W.omega(w), x.q, x.k, x.v,
                                           O.gate_rows(x.gate, w.kind, D), x.beta, scheme="row_absmax")
        pool.decode_step(slots_t(reqs), dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
        assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2, f"step {t}"
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    S_gpu = O.dequantize(ug, rg, cg, pg, rb)
    S_or = O.dequantize(u, r, c, piv, rb)
    assert T.rel_l2(S_gpu, S_or) <= T.CHAIN_REL_L2


# ---------------------------------------------------------------------------------
# compact pools: r and c stored as binary16 (both quantisers)
# ---------------------------------------------------------------------------------
def _quantiser(scheme):
    if scheme == "row_absmax":
        return lambda S, om, rb: O.absmax_quantise(S, rb, scale16=True)
    return lambda S, om, rb: O.refit(S, om, rb, scale16=True)


@pytest.mark.parametrize("widx", [1, 2])
@pytest.mark.parametrize("scheme", ["stepquant", "row_absmax"])
def test_scale16_quantize_step_and_chain(widx, scheme):
    w = W.WORKLOADS[widx]
    reqs = [0, w.B - 1]
    rb, om = W.row_bits(w), W.omega(w)
    pool = stq.Pool(w.kind, W.n_slots(w.B), W.unit_bits(w), om, scheme=scheme, scale_bits=16)
    L = O.Layout(rb)
    slots = [W.slot_of_request(b) for b in reqs]
    S0 = T.warm_state(w.index, tuple(reqs))
    # quantise: same codes and binary16 scales as the oracle
    u, r, c, piv = _quantiser(scheme)(S0, om, rb)
    pool.quantize_init(slots_t(reqs), dev(S0))
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u, S0, r, c, rb, "scale16 quantize_init", config=f"{w.name} {scheme} scale16")
    T.check_scales(rg, r, cg, c, n, "scale16 quantize_init", c_rel=2.0 ** -10)
    # chained steps from the oracle's packed state
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    for t in range(16):
        x = T.inputs_for(w, "decode", t, reqs)
        u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v,
                                             O.gate_rows(x.gate, w.kind, D), x.beta,
                                             scheme=scheme, scale16=True)
        pool.decode_step(slots_t(reqs), dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
        assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2, f"step {t}"
        if t == 0:     # teacher-forced first step: the step rule itself
            ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
            n = T.compare_codes(ug, u2, X, r2, c2, rb, "scale16 step", config=f"{w.name} {scheme} scale16")
            T.check_scales(rg, r2, cg, c2, n, "scale16 step", c_rel=2.0 ** -10)
        u, r, c, piv = u2, r2, c2, p2
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    assert T.rel_l2(O.dequantize(ug, rg, cg, pg, rb), O.dequantize(u, r, c, piv, rb)) <= T.CHAIN_REL_L2
    # the dequantiser reads binary16 scales
    Sd = torch.empty((len(reqs), w.H, D, D), device="cuda")
    pool.dequantize(slots_t(reqs), Sd)
    assert np.array_equal(Sd.cpu().numpy(), O.dequantize(ug, rg, cg, pg, rb))


# ---------------------------------------------------------------------------------
# every width on the uniform-width code paths (each head one width), both kinds
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("widx", [1, 2])
@pytest.mark.parametrize("bits", [2, 4, 6, 8])
def test_uniform_width_paths_step(widx, bits):
    w = W.WORKLOADS[widx]
    reqs = [0, 1]
    rb = np.full((w.H, D), bits)
    ub = np.full(w.H if w.kind == "gdn" else w.H * D, bits, np.uint8)
    om = W.omega(w)
    pool = stq.Pool(w.kind, 4, ub, om)
    L = O.Layout(rb)
    slots = [1, 3]
    S0 = T.warm_state(w.index, tuple(reqs))
    u, r, c, piv = O.refit(S0, om, rb)
    pool.quantize_init(torch.tensor(slots, dtype=torch.int32, device="cuda"), dev(S0))
    pool.check()
    ug, rg, cg, _ = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u, S0, r, c, rb, f"{bits}-bit quantize", config=f"{w.kind} uniform {bits}-bit")
    T.check_scales(rg, r, cg, c, n, f"{bits}-bit quantize")
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    x = T.inputs_for(w, "decode", 3, reqs)
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, rb, om, x.q, x.k, x.v,
                                         O.gate_rows(x.gate, w.kind, D), x.beta)
    out = torch.empty((2, w.H, D), device="cuda")
    pool.decode_step(torch.tensor(slots, dtype=torch.int32, device="cuda"), dev(x.q), dev(x.k), dev(x.v),
                     dev(x.gate), dev(x.beta), out)
    pool.check()
    ug, rg, cg, _ = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u2, X, r2, c2, rb, f"{bits}-bit step", config=f"{w.kind} uniform {bits}-bit")
    T.check_scales(rg, r2, cg, c2, n, f"{bits}-bit step")
    assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2


# ---------------------------------------------------------------------------------
# degenerate scales inside a head: zero rows and columns, rows whose scale falls below
# 2^-126 (their reciprocal counts as 0), a row five decades larger than the rest, and
# a head whose every row is below 2^-126 (c = 0: no least-squares denominator)
# ---------------------------------------------------------------------------------
def _degenerate_state(w, reqs):
    S = T.warm_state(w.index, tuple(reqs)).copy()
    rb = W.row_bits(w)
    heads = [h for h in range(w.H) if rb[h, 0] != 16][:2]
    h0, h1 = heads
    S[0, h0, [3, 40], :] = 0.0
    S[0, h0, :, [7, 100]] = 0.0
    S[0, h0, 50, :] *= F32(1e-39)           # subnormal row: r < 2^-126
    S[0, h0, 60, :] *= F32(1e5)             # (FP16 pivot rows stay finite after the step)
    S[0, h1] *= F32(1e-40)                  # every row below 2^-126
    return S, h0, h1


@pytest.mark.parametrize("widx", [1, 2])
@pytest.mark.parametrize("scheme", ["stepquant", "row_absmax"])
def test_degenerate_rows_and_columns(widx, scheme):
    w = W.WORKLOADS[widx]
    reqs = [0, w.B - 1]
    rb, om = W.row_bits(w), W.omega(w)
    pool = stq.Pool(w.kind, W.n_slots(w.B), W.unit_bits(w), om, scheme=scheme)
    L = O.Layout(rb)
    slots = [W.slot_of_request(b) for b in reqs]
    S0, h0, h1 = _degenerate_state(w, reqs)
    quantise = (lambda S: O.absmax_quantise(S, rb)) if scheme == "row_absmax" else (lambda S: O.refit(S, om, rb))
    u, r, c, piv = quantise(S0)
    assert np.all(r[0, h1] == 0) or np.all(r[0, h1] < np.float32(2.0 ** -126))
    pool.quantize_init(slots_t(reqs), dev(S0))
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u, S0, r, c, rb, "degenerate quantize_init", config=f"{w.kind} degenerate {scheme}")
    T.check_scales(rg, r, cg, c, n, "degenerate quantize_init")
    piv_rows = rb == 16
    assert np.array_equal(pg[:, piv_rows], piv[:, piv_rows])
    # one step from the oracle's packed state; k_i = 0 keeps the zero rows zero and
    # v_j = 0 (with u_j = 0) keeps the zero columns zero
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    x = T.inputs_for(w, "decode", 0, reqs)
    k = x.k.copy()
    v = x.v.copy()
    k[0, h0, [3, 40]] = 0.0
    v[0, h0, [7, 100]] = 0.0
    u2, r2, c2, p2, o, X = O.decode_step(u, r, c, piv, rb, om, x.q, k, v,
                                         O.gate_rows(x.gate, w.kind, D), x.beta, scheme=scheme)
    assert np.all(X[0, h0, [3, 40]] == 0) and np.all(X[0, h0][:, [7, 100]] == 0)
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    pool.decode_step(slots_t(reqs), dev(x.q), dev(k), dev(v), dev(x.gate), dev(x.beta), out)
    pool.check()
    ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
    n = T.compare_codes(ug, u2, X, r2, c2, rb, "degenerate step", config=f"{w.kind} degenerate {scheme}")
    T.check_scales(rg, r2, cg, c2, n, "degenerate step")
    assert np.array_equal(pg[:, piv_rows], p2[:, piv_rows])
    assert T.per_vector_rel_l2(out.cpu().numpy(), o).max() <= T.OUT_REL_L2
