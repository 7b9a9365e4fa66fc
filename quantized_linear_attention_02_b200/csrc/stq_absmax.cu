// Decode step and state quantisation with the pages' uniform comparison quantiser:
// symmetric per-key-row absmax INT-b (singularity-lens, calibration and
// evaluation-setup paragraphs). The restore, gated delta update and readout are the
// decode kernel's own (stq_device.cuh); only the quantiser that ends the step differs:
//   r_i = max_j |S_ij| * fl(1/qmax_i),  Q_ij = clamp(rint(S_ij * fl(1/r_i)), +-qmax_i),
//   c_j = 1,
// so the pool keeps the dual-axis layout and dequantises as (Q r) * 1. A row scale
// below 2^-126 counts as zero (all-zero codes), as in the method's refit.
#include "stq_device.cuh"

namespace stq {
namespace {

struct AbsmaxStore {
  template <int BITS, class Sc>
  static __device__ __forceinline__ void store(CtaSmem& cs, WarpRows& wr, f2 (&s)[RPW][2], const Sc& sc,
                                               uint8_t* codes_global, int warp_code_start, float* o_global,
                                               uint8_t* stage) {
    const int w = group_tid() >> 5, lane = group_tid() & 31;
    const int r0 = w * RPW;

    // --- row maxima of |S| (exact in any order): 4 columns per lane, then across the
    // lanes -------------------------------------------------------------------------
    float a[RPW];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr)
      a[rr] = fmaxf(fmaxf(fabsf(s[rr][0].x), fabsf(s[rr][0].y)), fmaxf(fabsf(s[rr][1].x), fabsf(s[rr][1].y)));
    // through the warp's consumed code staging area, as the refit's row sums: lane l
    // writes its 16 row maxima at tr[rr][l ^ 4 (rr & 7)], lane L takes row L & 15 over
    // lanes 16 (L >> 4) .. +15, and the two halves meet in one shuffle
    float* tr = reinterpret_cast<float*>(stage);
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) tr[rr * 32 + (lane ^ (4 * (rr & 7)))] = a[rr];
    __syncwarp();
    {
      const int Rr = lane & 15, hh = lane >> 4;
      float m = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(tr + Rr * 32 + ((16 * hh + 4 * j) ^ (4 * (Rr & 7))));
        m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
      }
      a[0] = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
    }
    __syncwarp();   // the staging area is free again
    {
      const int R = lane & 15;   // lane l holds the maximum of row l & 15
      float iq;
      bool pivot = false;
      if constexpr (BITS == MIXED) {
        iq = wr.iq[R];
        pivot = row_bits(wr.info[R]) == PIVOT;
      } else {
        iq = __frcp_rn(float((1 << (BITS - 1)) - 1));
      }
      const float r = sc.stored(pivot ? 0.0f : fmul(a[0], iq));   // codes fit the stored r
      if (lane < 16) {
        const float ir = recip_scale(r);
        wr.irr[R] = make_float2(ir, ir);
        sc.put(r0 + R, r);
      }
    }
    if (lane < 16) sc.put(D + 16 * w + lane, 1.0f);
    __syncwarp();

    // --- codes: x = S * (1/r_i) taken exactly, rounded in the 2^23 binade ---------
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const float4 i2 = *reinterpret_cast<const float4*>(&wr.irr[rr & ~1]);
      const f2 ir = (rr & 1) ? make_float2(i2.z, i2.w) : make_float2(i2.x, i2.y);
      // |S_ij| * fl(1/r_i) <= qmax (1 + 2^-22) (binary16 r: <= qmax (1 + 2^-10)), so
      // |n| <= qmax + 1: the 16-bit lanes hold it
      if constexpr (BITS == MIXED) {
        // the refit's branch-free staged store (a pivot row stores nothing)
        const uint4 T = wr.st[rr];
        const f2 mb = dup(__uint_as_float(T.x));
        stage_mixed_codes(T, fma2(s[rr][0], ir, mb), fma2(s[rr][1], ir, mb),
                          static_cast<uint32_t>(__cvta_generic_to_shared(stage)), lane);
      } else {
        constexpr float MB = MAGIC + float(1 << (BITS - 1));
        constexpr uint32_t HI = ((1u << BITS) - 1u) * 0x00010001u;
        const f2 t01 = fma2(s[rr][0], ir, dup(MB));
        const f2 t23 = fma2(s[rr][1], ir, dup(MB));
        store_codes_s16<BITS>(codes_global + warp_code_start + rr * (D * BITS / 8), lane, t01, t23, HI);
      }
    }
    if constexpr (BITS == MIXED) copy_out_staged(wr, stage, codes_global + warp_code_start, lane);

    // --- readout from the per-warp partials the caller left in red[1][0] ------------
    if (o_global != nullptr) {
      group_sync();
      if (w == 0) {
        f2 lo, hi;
        warp_tree(cs.red[1][0], lane, lo, hi);
        *reinterpret_cast<float4*>(o_global + 4 * lane) = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
    }
  }
};

}  // namespace

cudaError_t launch_decode_absmax(const PoolDev& P, const int32_t* slots, int B, const float* q,
                                 const float* k, const float* v, const float* gate,
                                 const float* beta, float* out, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const unsigned n = unsigned(B) * unsigned(P.H);
  constexpr int SM = 2 * sizeof(DecodeSmem);
  if (P.scale16) {
    if (P.any_mixed) return launch_persistent<decode_kernel<AbsmaxStore, true, true>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
    return launch_persistent<decode_kernel<AbsmaxStore, false, true>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
  }
  if (P.any_mixed) return launch_persistent<decode_kernel<AbsmaxStore, true, false>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
  return launch_persistent<decode_kernel<AbsmaxStore, false, false>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
}

cudaError_t launch_quantize_absmax(const PoolDev& P, const int32_t* slots, int B, const float* S,
                                   cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const unsigned n = unsigned(B) * unsigned(P.H);
  constexpr int SM = sizeof(CtaSmem);
  if (P.scale16) return launch_items<quantize_kernel<AbsmaxStore, true>>(n, SM, s, P, slots, B, S);
  return launch_items<quantize_kernel<AbsmaxStore, false>>(n, SM, s, P, slots, B, S);
}

}  // namespace stq
