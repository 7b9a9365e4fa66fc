"""The decode step is capture-safe: recorded once into a CUDA graph and replayed, it
gives bit for bit the states and readouts of the same steps launched one by one (the
entry point only enqueues a kernel on the caller's stream: no allocation, no sync)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from oracle import stq_oracle as O  # noqa: E402
from quantized_linear_attention_02_b200 import build, stq  # noqa: E402
from quantized_linear_attention_02_b200 import workload as W  # noqa: E402

D = 128


@pytest.mark.parametrize("widx", [1, 2])
def test_graph_replay_matches_eager_steps(widx):
    build.build()
    w = W.WORKLOADS[widx]
    B, steps = 4, 6
    ub, om = W.unit_bits(w), W.omega(w)
    pools = [stq.Pool(w.kind, B, ub, om) for _ in range(2)]
    slots = torch.arange(B, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    S0 = torch.randn(B, w.H, D, D, device="cuda", generator=g) * 0.1
    for p in pools:
        p.quantize_init(slots, S0)
    gen = torch.Generator(device="cuda").manual_seed(8)
    inputs = [W.torch_step_inputs(w, B, gen, "cuda") for _ in range(steps)]
    # eager
    outs_e = []
    for x in inputs:
        o = torch.empty(B, w.H, D, device="cuda")
        pools[0].decode_step(slots, *x, o)
        outs_e.append(o)
    # graph: static input/output buffers, one captured step replayed per input set
    static_in = [t.clone() for t in inputs[0]]
    static_out = torch.empty(B, w.H, D, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        pools[1].decode_step(slots, *static_in, static_out, stream=side)
    # capture recorded the launch without running it: the pool is still at S0
    outs_g = []
    for x in inputs:
        for dst, src in zip(static_in, x):
            dst.copy_(src)
        graph.replay()
        outs_g.append(static_out.clone())
    torch.cuda.synchronize()
    for p in pools:
        p.check()
    for a, b in zip(outs_e, outs_g):
        assert torch.equal(a, b)
    L = O.Layout(W.row_bits(w))
    img = [O.Pool(L, B) for _ in range(2)]
    for p, im in zip(pools, img):
        im.codes[:] = p.codes_view().cpu().numpy()
        im.scales[:] = p.scales_view().cpu().numpy()
        if L.n_pivot_rows:
            im.pivots[:] = p.pivots_view().cpu().numpy()
    assert np.array_equal(img[0].codes, img[1].codes)
    assert np.array_equal(img[0].scales, img[1].scales)
    assert np.array_equal(img[0].pivots, img[1].pivots)
