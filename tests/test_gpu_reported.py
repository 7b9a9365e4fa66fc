"""Measurements of the CUDA path that are reported, not gated (printed at the end of the
pytest run):
  * the drift of the KDA throughput workload (B = 512, H = 32, nominal 6-bit rows,
    FP16 pivot rows) from the oracle over 1,024 chained decode steps of one request
    inside the full-B launch;
  * the distance of the GPU chain from the plain float64 statement of the rule
    (oracle/plain_rule.py) over 64 chained steps of the GDN parity workload.
Both sides of each comparison start from one packed state and then run on their own,
so the numbers measure how far two quantised chains drift apart, not a per-step
error."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from oracle import plain_rule as P  # noqa: E402
from oracle import stq_oracle as O  # noqa: E402
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


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def test_kda_throughput_workload_1024_step_drift_from_oracle():
    import concurrent.futures as cf
    import multiprocessing as mp
    widx, steps, marks = 4, 1024, (64, 256, 1024)
    w = W.WORKLOADS[widx]
    rb, om = W.row_bits(w), W.omega(w)
    b = int(W.parity_sample(w, 1)[0])
    pool = stq.Pool(w.kind, W.n_slots(w.B), W.unit_bits(w), om)
    L = O.Layout(rb)
    S0 = T.warm_states(widx, [b])
    u, r, c, piv = O.refit(S0, om, rb)
    g = torch.Generator(device="cuda").manual_seed(4)
    S_all = torch.randn((w.B, w.H, D, D), device="cuda", generator=g) * 0.05
    all_slots = torch.tensor([W.slot_of_request(i) for i in range(w.B)], dtype=torch.int32, device="cuda")
    pool.quantize_init(all_slots, S_all)
    del S_all
    slot = W.slot_of_request(b)
    T.write_oracle_state(pool, L, [slot], u, r, c, piv)
    # the oracle's chain runs in a worker process while the GPU steps
    with cf.ProcessPoolExecutor(1, mp_context=mp.get_context("spawn")) as ex:
        fut = ex.submit(T.oracle_chain, widx, b, (u, r, c, piv), 0, steps, marks)
        gen = torch.Generator(device="cuda").manual_seed(5)
        out = torch.empty((w.B, w.H, D), device="cuda")
        o_gpu, S_gpu = [], {}
        one = torch.tensor([slot], dtype=torch.int32, device="cuda")
        Sg = torch.empty((1, w.H, D, D), device="cuda")
        for t in range(steps):
            xin = list(W.torch_step_inputs(w, w.B, gen, "cuda"))
            xs = W.step_inputs(w, "decode", t, b, b + 1)
            for a, name in zip(xin, ("q", "k", "v", "gate", "beta")):
                a[b] = dev(getattr(xs, name)[0])
            pool.decode_step(all_slots, *xin, out)
            o_gpu.append(out[b].cpu().numpy())
            if t + 1 in marks:
                pool.dequantize(one, Sg)
                S_gpu[t + 1] = Sg[0].cpu().numpy()
        pool.check()
        o_or, _, S_or = fut.result()
    o_gpu = np.stack(o_gpu)
    parts = []
    for m in marks:
        rel_s = T.rel_l2(S_gpu[m], S_or[m])
        rel_o = float(T.per_vector_rel_l2(o_gpu[:m], o_or[:m]).max())
        parts.append(f"after {m} steps state rel L2 {rel_s:.3g}, worst readout rel L2 {rel_o:.3g}")
        assert np.isfinite(rel_s) and np.isfinite(rel_o)
    T.REPORTS[f"{w.name} request {b}, GPU vs oracle chains"] = "; ".join(parts)


def test_gpu_chain_against_plain_float64_rule():
    """How far the shipped float32 arithmetic sits from the plain float64 statement of
    the rule along a chain: the step at which a code first differs, then the fraction of
    codes that differ and the distance of the dequantised states at a few steps, next
    to the distance of each chain from the unquantised FP32 state (the chains' own
    quantisation error, the scale against which their distance is read)."""
    widx, steps, marks = 1, 64, (1, 2, 4, 8, 16, 32, 64)
    w = W.WORKLOADS[widx]
    rb, om = W.row_bits(w), W.omega(w)
    reqs = [1, w.B - 2]
    pool = stq.Pool(w.kind, W.n_slots(w.B), W.unit_bits(w), om)
    L = O.Layout(rb)
    S0 = T.warm_state(widx, tuple(reqs))
    u, r, c, piv = O.refit(S0, om, rb)
    slots = [W.slot_of_request(b) for b in reqs]
    T.write_oracle_state(pool, L, slots, u, r, c, piv)
    st = torch.tensor(slots, dtype=torch.int32, device="cuda")
    out = torch.empty((len(reqs), w.H, D), device="cuda")
    pu, pr, pc, pp = u, r.astype(np.float64), c.astype(np.float64), piv
    S_fp = O.dequantize(u, r, c, piv, rb).astype(np.float64)
    quant = np.broadcast_to((rb != 16)[..., None], u.shape)
    first, parts = None, []
    for t in range(steps):
        x = T.inputs_for(w, "decode", t, reqs)
        dec = O.gate_rows(x.gate, w.kind, D)
        Q, pr, pc, pp, o, _ = P.decode_step(pu, pr, pc, pp, rb, om, x.q, x.k, x.v, dec, x.beta)
        pu = P.biased_codes(Q, rb)
        S_fp = P.gated_delta_update(S_fp, x.k, x.v, dec, x.beta)
        pool.decode_step(st, dev(x.q), dev(x.k), dev(x.v), dev(x.gate), dev(x.beta), out)
        ug, rg, cg, pg = T.read_pool_state(pool, L, slots)
        n_diff = int(((ug != pu) & quant).sum())
        if first is None and n_diff:
            first = t + 1
        if t + 1 in marks:
            S_gpu = O.dequantize(ug, rg, cg, pg, rb).astype(np.float64)
            S_plain = P.restore(pu, pr, pc, pp, rb)
            parts.append(f"step {t + 1}: codes differing {n_diff / quant.sum():.3g}, "
                         f"GPU-plain {T.rel_l2(S_gpu, S_plain):.3g}, "
                         f"GPU-FP32 {T.rel_l2(S_gpu, S_fp):.3g}, plain-FP32 {T.rel_l2(S_plain, S_fp):.3g}")
    pool.check()
    T.REPORTS[f"{w.name} 2 requests, GPU vs plain float64 rule (state rel L2)"] = (
        f"first code difference at step {first}; " + "; ".join(parts))
    assert first is None or first >= 1
