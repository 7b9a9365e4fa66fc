"""CPU oracle for the packed Delta-rule state decode step (test infrastructure).

This package is the plain, slow, obviously-correct restatement of what the decode
step computes (and of the offline bit allocation before it). It is used only by the
tests, by `__graft_entry__.smoke()` and by the `cpu_baseline` / `--impl reference`
legs of `bench.py`. The library's product path
never imports, links or runs anything here, and nothing here imports the library:
the two share no code, tables or constants. Only the seeded input generator
(`quantized_linear_attention_02_b200.workload`, which holds none of the method's
arithmetic) feeds both sides.

Source: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
Quantization" (arXiv 2609.38169), as five web pages render it. Each function in
`stq_oracle` names the passage it follows.

Parity status per function (what pins it, see tests/test_oracle_*.py):
  pack_row / unpack_row     pinned (hand-written byte vectors, round trip)
  row_gain                  pinned (closed form on square ratios)
  dequantize                pinned (hand example, closed form)
  fp32_update / readout     pinned (literal fp64 matrix form of the gated delta rule,
                            delta property, beta=0 identity, spectral bound)
  refit (quantiser)         pinned (exact-rational brute force on tiny states,
                            half-step bound, no clipping at c0, weighted
                            least-squares optimality vs numpy lstsq, scaling and
                            sign symmetry, rank-1 fixed point)
  decode_step               pinned (error recurrence on paired FP32 / quantised runs,
                            readout taken before requantisation, all-pivot tracking)
  absmax_quantise           pinned (row maximum to +-qmax, half-step bound, float64
                            textbook absmax quantiser, symmetry, hand example)
  stq_alloc.lifetime_weight pinned (closed form of the geometric series)
  stq_alloc.allocate        pinned (brute force over all width choices on tiny
                            instances, pivots = riskiest units, budget limits)
  stq_alloc.row_sq_error,
  stq_alloc.unit_distortion pinned (float64 numpy means; distortion falls with width)
The refit rule itself (which scales the paper's authors use) is not printed on the
pages; the rule here is the documented build rule, so agreement with the authors'
own quantiser is unpinned.
"""
