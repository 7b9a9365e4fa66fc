// Kernels of the packed Delta-rule state decode step for B200 (sm_100a).
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
// Quantization" (arXiv 2609.38169) as its web pages describe it -- gated delta rule
// (bloombook.cn tutorial, section 2), readout before requantisation (singularity-lens
// summary, decode-order paragraph), dual-axis scales r_i c_j z_ij (bloombook section 4),
// per-unit widths and FP16 pivot units (ai-trend review, Method).
//
// A group of 256 threads (8 warps) owns one (request, head) 128x128 state at a time
// (the decode kernel runs two such groups per CTA on separate items; the others one per
// CTA). Warp w holds key rows 16w..16w+15, lane l holds value columns 4l..4l+3 as two
// float2 pairs, so a thread keeps 64 state values in registers for the whole step. A
// row's width is uniform across a warp instruction (KDA widths vary per key row without
// divergence); heads whose rows share one width run a code path specialised for it.
//
// Float32 evaluation order of every sum that decides a code or a scale (the CPU oracle
// restates the same order):
//   * sums over the 128 rows of a column or the 128 columns of a row are balanced
//     binary trees, adjacent pairs first. Column sums: a thread's 16 rows form the
//     lower 4 levels, the 8 warps (shared memory) the top 3. Row sums: a thread's 4
//     columns form the lower 2 levels, then 16 lanes' partials (a shared-memory
//     transpose) the next 4 and one shuffle between the two halves of the warp the top;
//   * in a sum of products a_i b_i each adjacent pair is one fused multiply-add,
//     fma(a_2m, b_2m, a_2m+1 * b_2m+1); the state update is S = fma(k, delta, S'); every
//     other product is rounded on its own (explicit _rn forms, --fmad=false);
//   * the quantiser's x = y * inv_c is taken exactly: fma(y, inv_c, 1.5*2^23) rounds the
//     exact product to the nearest integer (ties to even) inside the 2^23 binade, where
//     the low bits are the (biased) code; the least-squares step clamps in that binade,
//     the final codes clamp in 16-bit lanes (same result, see refit_store).
//
// The readout is compared within a tolerance, not bit for bit; each warp forms its
// partials as running sums. This file holds the dual-axis refit (the quantiser of the
// method), the dequantise and FP32-state kernels and the launchers; the kernel bodies
// shared with the row-absmax baseline are in stq_device.cuh.
#include "stq_device.cuh"

namespace stq {
namespace {

// ---------------------------------------------------------------------------------
// Refit of this warp's rows: row scale, column scale start, two omega-weighted
// least-squares steps, final codes (bloombook section 4; singularity-lens dual-axis
// paragraph). On entry s[][] holds the float32 state (pivot rows already stored) and the
// caller may have put readout partials into red[1][0]. The codes go straight to the
// pool; r of this warp's rows and c of the columns this warp owns are written.
// Five CTA barriers: column maximum, and per least-squares step one for the partial sums
// and one for the new 1/c.
// ---------------------------------------------------------------------------------
template <int BITS, class Sc>
__device__ __forceinline__ void refit_store(CtaSmem& cs, WarpRows& wr, f2 (&s)[RPW][2], const Sc& sc,
                                            uint8_t* codes_global, int warp_code_start, float* o_global,
                                            uint8_t* stage) {
  const int w = group_tid() >> 5, lane = group_tid() & 31;
  const int r0 = w * RPW;

  // --- row scale r_i = (tree sum_j |S_ij|) / 128 * g_i -------------------------------
  float a[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr)
    a[rr] = fadd(fadd(fabsf(s[rr][0].x), fabsf(s[rr][0].y)), fadd(fabsf(s[rr][1].x), fabsf(s[rr][1].y)));
  // Row sums through the warp's consumed code staging area: lane l writes its 16 row
  // partials at tr[rr][l ^ 4 (rr & 7)] (the swizzle keeps every group of 4 lanes whole and
  // spreads the rows over the banks); lane L then adds row L & 15 over lanes 16 (L >> 4)
  // .. +15 as a balanced tree, and the two halves meet in one shuffle: the same tree over
  // the 128 columns as lane pairs xor 1, 2, 4, 8, 16 would make.
  float* tr = reinterpret_cast<float*>(stage);
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) tr[rr * 32 + (lane ^ (4 * (rr & 7)))] = a[rr];
  __syncwarp();
  {
    const int Rr = lane & 15, hh = lane >> 4;
    float p[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(tr + Rr * 32 + ((16 * hh + 4 * j) ^ (4 * (Rr & 7))));
      p[4 * j] = v.x; p[4 * j + 1] = v.y; p[4 * j + 2] = v.z; p[4 * j + 3] = v.w;
    }
#pragma unroll
    for (int m = 1; m < 16; m <<= 1)
#pragma unroll
      for (int t = 0; t < 16; t += 2 * m) p[t] = fadd(p[t], p[t + m]);
    a[0] = fadd(p[0], __shfl_xor_sync(0xffffffffu, p[0], 16));
  }
  __syncwarp();   // the staging area is free again
  {
    // lane l holds the sum of row l & 15
    const int R = lane & 15;
    const bool pivot = (BITS == MIXED) ? (row_bits(wr.info[R]) == PIVOT) : false;
    // a compact pool rounds r to binary16 here: y, the weights and the codes use it
    const float r = sc.stored(pivot ? 0.0f : fmul(fmul(a[0], 0.0078125f), wr.g[R]));
    if (lane < 16) {
      const float ir = recip_scale(r), bv = fmul(wr.om[R], fmul(r, r));
      wr.irr[R] = make_float2(ir, ir);
      wr.bb[R] = make_float2(bv, bv);
      sc.put(r0 + R, r);
    }
  }
  __syncwarp();

  // --- y = S * inv_r; column start c0_j = max_i |y_ij| / qmax_i -----------------------
  float mx[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const float4 i2 = *reinterpret_cast<const float4*>(&wr.irr[rr & ~1]);
    const f2 ir = (rr & 1) ? make_float2(i2.z, i2.w) : make_float2(i2.x, i2.y);
    s[rr][0] = mul2(s[rr][0], ir);
    s[rr][1] = mul2(s[rr][1], ir);
    if constexpr (BITS == MIXED) {
      // |y| / qmax_i as |y * fl(1/qmax_i)| (rounding is symmetric)
      const f2 iq = dup(wr.iq[rr]);
      const f2 p01 = mul2(s[rr][0], iq), p23 = mul2(s[rr][1], iq);
      mx[0] = fmaxf(mx[0], fabsf(p01.x));
      mx[1] = fmaxf(mx[1], fabsf(p01.y));
      mx[2] = fmaxf(mx[2], fabsf(p23.x));
      mx[3] = fmaxf(mx[3], fabsf(p23.y));
    } else {
      mx[0] = fmaxf(mx[0], fabsf(s[rr][0].x));
      mx[1] = fmaxf(mx[1], fabsf(s[rr][0].y));
      mx[2] = fmaxf(mx[2], fabsf(s[rr][1].x));
      mx[3] = fmaxf(mx[3], fabsf(s[rr][1].y));
    }
  }
  cs.red[1][1][w][lane] = make_float4(mx[0], mx[1], mx[2], mx[3]);
  group_sync();

  if (o_global != nullptr && w == 0) {
    f2 lo, hi;
    warp_tree(cs.red[1][0], lane, lo, hi);
    *reinterpret_cast<float4*>(o_global + 4 * lane) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  // Column scales are owned: lane l of warp w (l < 16) owns column 16w + l, keeps its c
  // in a register and publishes 1/c for everyone through shared memory; the other 16
  // lanes help reduce the least-squares denominators.
  const int jown = 16 * w + (lane & 15);
  float c_own;
  {
    float m = 0.0f;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) m = fmaxf(m, reinterpret_cast<const float*>(cs.red[1][1][ww])[jown]);
    if constexpr (BITS != MIXED) {
      // max_i RN(|y| / qmax) = RN(max_i |y| / qmax): rounding is monotone
      constexpr float QM = float((1 << (BITS - 1)) - 1);
      m = fmul(m, __frcp_rn(QM));
    }
    c_own = m;
    const float ic0 = recip_scale(c_own);
    if (lane < 16) cs.col_ic[jown] = ic0;
  }
  const float c0 = c_own;
  int wide = 0, any_wide = 0;
  group_sync();

  // --- two least-squares steps: c_j <- sum_i p y / sum_i p Q, p = b_i Q_ij -------------
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    f2 ic[2];
    {
      const float4 i4 = *reinterpret_cast<const float4*>(&cs.col_ic[4 * lane]);
      ic[0] = make_float2(i4.x, i4.y);
      ic[1] = make_float2(i4.z, i4.w);
    }
    V2<4> nd = tree<0, RPW / 2, 4>([&](int m) {
      // rows 2m and 2m+1 form one fused pair of each sum
      f2 Q[2][2], p[2][2];
      const float4 b2 = *reinterpret_cast<const float4*>(&wr.bb[2 * m]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int rr = 2 * m + e;
        const f2 bb = e == 0 ? make_float2(b2.x, b2.y) : make_float2(b2.z, b2.w);
        float lo_b, hi_b;
        if constexpr (BITS == MIXED) {
          const f2 cb = wr.clampb[rr];
          lo_b = cb.x;
          hi_b = cb.y;
        } else {
          lo_b = MAGIC - float((1 << (BITS - 1)) - 1);
          hi_b = MAGIC + float((1 << (BITS - 1)) - 1);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          f2 t = fma2(s[rr][hh], ic[hh], dup(MAGIC));
          if (it > 0) {  // step one never clips: c0 is the column maximum
            t.x = fminf(fmaxf(t.x, lo_b), hi_b);
            t.y = fminf(fmaxf(t.y, lo_b), hi_b);
          }
          Q[e][hh] = add2(t, dup(-MAGIC));
          p[e][hh] = mul2(bb, Q[e][hh]);
        }
      }
      V2<4> leaf;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        leaf.x[hh] = fma2(p[0][hh], s[2 * m][hh], mul2(p[1][hh], s[2 * m + 1][hh]));
        leaf.x[2 + hh] = fma2(p[0][hh], Q[0][hh], mul2(p[1][hh], Q[1][hh]));
      }
      return leaf;
    });
    put_partial(cs.red[it][0], w, lane, nd.x[0], nd.x[1]);
    put_partial(cs.red[it][1], w, lane, nd.x[2], nd.x[3]);
    group_sync();
    {
      // lanes 0..15: numerator of column jown, lanes 16..31: its denominator
      const float* part = reinterpret_cast<const float*>(cs.red[it][lane >> 4][0]);
      float x[NW];
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) x[ww] = part[ww * D + jown];
      const float sum = fadd(fadd(fadd(x[0], x[1]), fadd(x[2], x[3])), fadd(fadd(x[4], x[5]), fadd(x[6], x[7])));
      const float den = __shfl_down_sync(0xffffffffu, sum, 16);
      // lanes 16..31 compute a value they never store (no divergent branch)
      const float q = __fdiv_rn(sum, den);
      if (den > 0.0f) c_own = q;
      if (it == 1) c_own = sc.stored(c_own);   // the final c as the pool will hold it
      const float icn = recip_scale(c_own);
      if (lane < 16) cs.col_ic[jown] = icn;
      // every least-squares step keeps c >= c_before / 2 (each term Q y >= c Q^2 / 2),
      // so |n| = |rint(y / c)| <= qmax c0 / c + 1/2 < 2^15 unless rounding at the bottom
      // of the float32 range broke that; then the column takes the float clamp
      if (it == 1) wide = lane < 16 && !(fmul(c0, icn) < 128.0f);
    }
    if (it == 1) any_wide = group_sync_or(wide);
    else group_sync();
  }

  // --- final codes with the final c, stored straight into the pool -------------------
  f2 ic[2];
  {
    const float4 i4 = *reinterpret_cast<const float4*>(&cs.col_ic[4 * lane]);
    ic[0] = make_float2(i4.x, i4.y);
    ic[1] = make_float2(i4.z, i4.w);
  }
  if (lane < 16) sc.put(D + jown, c_own);
  if constexpr (BITS != MIXED) {
    if (!any_wide) {
      constexpr float MB = MAGIC + float(1 << (BITS - 1));
      constexpr uint32_t HI = ((1u << BITS) - 1u) * 0x00010001u;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const f2 t01 = fma2(s[rr][0], ic[0], dup(MB));
        const f2 t23 = fma2(s[rr][1], ic[1], dup(MB));
        store_codes_s16<BITS>(codes_global + warp_code_start + rr * (D * BITS / 8), lane, t01, t23, HI);
      }
      return;
    }
  } else {
    if (!any_wide) {
      // Mixed widths: clamp in 16-bit lanes, pack any width without a branch, and put
      // each lane's b/2 bytes into the warp's staging area (the staged codes are consumed
      // by now), then copy the area out with 16-byte stores.
      const uint32_t stage_s = static_cast<uint32_t>(__cvta_generic_to_shared(stage));
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const uint4 T = wr.st[rr];
        const f2 mb = dup(__uint_as_float(T.x));
        stage_mixed_codes(T, fma2(s[rr][0], ic[0], mb), fma2(s[rr][1], ic[1], mb), stage_s, lane);
      }
      copy_out_staged(wr, stage, codes_global + warp_code_start, lane);
      return;
    }
  }
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    if constexpr (BITS == MIXED) {
      const uint32_t info = wr.info[rr];
      const int bits = row_bits(info);
      if (bits == PIVOT) continue;
      const float mb = wr.mb[rr], q = wr.qm[rr];
      const f2 t01 = fma2(s[rr][0], ic[0], dup(mb));
      const f2 t23 = fma2(s[rr][1], ic[1], dup(mb));
      const float lo_b = mb - q, hi_b = mb + q;
      const uint32_t t[4] = {__float_as_uint(fminf(fmaxf(t01.x, lo_b), hi_b)),
                             __float_as_uint(fminf(fmaxf(t01.y, lo_b), hi_b)),
                             __float_as_uint(fminf(fmaxf(t23.x, lo_b), hi_b)),
                             __float_as_uint(fminf(fmaxf(t23.y, lo_b), hi_b))};
      uint8_t* row = codes_global + row_off(info);
      switch (bits) {
        case 2: store_codes<2>(row, lane, t); break;
        case 4: store_codes<4>(row, lane, t); break;
        case 6: store_codes<6>(row, lane, t); break;
        default: store_codes<8>(row, lane, t); break;
      }
    } else {
      constexpr float MB = MAGIC + float(1 << (BITS - 1));
      constexpr float QM = float((1 << (BITS - 1)) - 1);
      const f2 t01 = fma2(s[rr][0], ic[0], dup(MB));
      const f2 t23 = fma2(s[rr][1], ic[1], dup(MB));
      const uint32_t t[4] = {__float_as_uint(fminf(fmaxf(t01.x, MB - QM), MB + QM)),
                             __float_as_uint(fminf(fmaxf(t01.y, MB - QM), MB + QM)),
                             __float_as_uint(fminf(fmaxf(t23.x, MB - QM), MB + QM)),
                             __float_as_uint(fminf(fmaxf(t23.y, MB - QM), MB + QM))};
      store_codes<BITS>(codes_global + warp_code_start + rr * (D * BITS / 8), lane, t);
    }
  }
}

// The quantiser of the method: dual-axis refit (refit_store).
struct StepQuantStore {
  template <int BITS, class Sc>
  static __device__ __forceinline__ void store(CtaSmem& cs, WarpRows& wr, f2 (&s)[RPW][2], const Sc& sc,
                                               uint8_t* codes, int warp_code_start, float* o, uint8_t* stage) {
    refit_store<BITS>(cs, wr, s, sc, codes, warp_code_start, o, stage);
  }
};

// ---------------------------------------------------------------------------------
// stq_dequantize: packed pool -> float32 states, S_ij = (Q_ij r_i) c_j.
// ---------------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ void dequant_row(const uint8_t* row, int lane, float r, const f2 (&cin)[2],
                                            float* dst) {
  f2 a, b;
  restore_row<BITS>(row, lane, r, cin, a, b);
  *reinterpret_cast<float4*>(dst) = make_float4(a.x, a.y, b.x, b.y);
}

template <bool H16>
__global__ void __launch_bounds__(NT)
dequant_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, float* __restrict__ S_out) {
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ uint32_t info_s[D];
  __shared__ float r_s[D];
  const int item = blockIdx.x;
  const int bq = item / P.H, h = item - bq * P.H;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int slot = slots[bq];
  if (slot < 0 || slot >= P.n_slots) {
    if (tid == 0) atomicOr(P.err, ERR_SLOT_RANGE);
    return;
  }
  const HeadRef<H16> hr = head_ref<H16>(P, slot, h);
  if (tid < D) {
    info_s[tid] = P.row_info[h * D + tid];
    r_s[tid] = hr.sc.get(tid);
  }
  copy16(stage, hr.codes, hr.code_bytes);
  copy16(stage + hr.piv_stage_off, hr.pivots, hr.piv_count * D * 2);
  const float4 c4 = hr.sc.get4(D + 4 * lane);
  const f2 cin[2] = {make_float2(c4.x, c4.y), make_float2(c4.z, c4.w)};
  __syncthreads();
  float* dst = S_out + uint64_t(item) * D * D;
#pragma unroll 4
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const uint32_t info = info_s[i];
    const uint8_t* row = stage + row_off(info);
    float* o = dst + i * D + 4 * lane;
    switch (row_bits(info)) {
      case 2: dequant_row<2>(row, lane, r_s[i], cin, o); break;
      case 4: dequant_row<4>(row, lane, r_s[i], cin, o); break;
      case 6: dequant_row<6>(row, lane, r_s[i], cin, o); break;
      case 8: dequant_row<8>(row, lane, r_s[i], cin, o); break;
      default: {
        const uint2 hv = *reinterpret_cast<const uint2*>(stage + hr.piv_stage_off + row_off(info) * (D * 2) + 8 * lane);
        f2 a, b;
        half4_floats(hv, a, b);
        *reinterpret_cast<float4*>(o) = make_float4(a.x, a.y, b.x, b.y);
      }
    }
  }
}

// ---------------------------------------------------------------------------------
// stq_fp32_decode_step: the unquantised FP32 state step, in place.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 2)
fp32_step_kernel(int kind, float* __restrict__ S, const float* __restrict__ q,
                 const float* __restrict__ k, const float* __restrict__ v,
                 const float* __restrict__ gate, const float* __restrict__ beta,
                 float* __restrict__ out) {
  __shared__ __align__(16) float ks[D], qs[D], vs[D], ds[D];
  __shared__ float4 red[2][NW][D / 4];
  const int item = blockIdx.x;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int r0 = w * RPW;
  const uint64_t vec = uint64_t(item) * D;
  if (tid < D) {
    ks[tid] = k[vec + tid];
    qs[tid] = q[vec + tid];
    vs[tid] = v[vec + tid];
    ds[tid] = (kind == 0) ? gate[item] : gate[vec + tid];
  }
  const float bt = beta[item];
  __syncthreads();
  float* base = S + vec * D;
  f2 s[RPW][2];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = r0 + rr;
    const float4 x = *reinterpret_cast<const float4*>(base + i * D + 4 * lane);
    const f2 dd = dup(ds[i]);
    s[rr][0] = mul2(dd, make_float2(x.x, x.y));
    s[rr][1] = mul2(dd, make_float2(x.z, x.w));
  }
  V2<2> u = tree<0, RPW / 2, 2>([&](int m) {
    const f2 ke = dup(ks[r0 + 2 * m]), ko = dup(ks[r0 + 2 * m + 1]);
    V2<2> leaf;
    leaf.x[0] = fma2(ke, s[2 * m][0], mul2(ko, s[2 * m + 1][0]));
    leaf.x[1] = fma2(ke, s[2 * m][1], mul2(ko, s[2 * m + 1][1]));
    return leaf;
  });
  put_partial(red[0], w, lane, u.x[0], u.x[1]);
  __syncthreads();
  f2 delta[2];
  {
    f2 ulo, uhi;
    warp_tree(red[0], lane, ulo, uhi);
    const float4 v4 = *reinterpret_cast<const float4*>(&vs[4 * lane]);
    delta[0] = mul2(dup(bt), add2(make_float2(v4.x, v4.y), make_float2(-ulo.x, -ulo.y)));
    delta[1] = mul2(dup(bt), add2(make_float2(v4.z, v4.w), make_float2(-uhi.x, -uhi.y)));
  }
  V2<2> o = tree<0, RPW / 2, 2>([&](int m) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int rr = 2 * m + e, i = r0 + rr;
      const f2 kk = dup(ks[i]);
      s[rr][0] = fma2(kk, delta[0], s[rr][0]);
      s[rr][1] = fma2(kk, delta[1], s[rr][1]);
      *reinterpret_cast<float4*>(base + i * D + 4 * lane) = make_float4(s[rr][0].x, s[rr][0].y, s[rr][1].x, s[rr][1].y);
    }
    const f2 qe = dup(qs[r0 + 2 * m]), qo = dup(qs[r0 + 2 * m + 1]);
    V2<2> leaf;
    leaf.x[0] = fma2(qe, s[2 * m][0], mul2(qo, s[2 * m + 1][0]));
    leaf.x[1] = fma2(qe, s[2 * m][1], mul2(qo, s[2 * m + 1][1]));
    return leaf;
  });
  put_partial(red[1], w, lane, o.x[0], o.x[1]);
  __syncthreads();
  if (w == 0) {
    f2 lo, hi;
    warp_tree(red[1], lane, lo, hi);
    *reinterpret_cast<float4*>(out + vec + 4 * lane) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
}

int stage_bytes(const PoolDev& P) { return (P.max_head_bytes + 15) & ~15; }

// Raise a kernel's dynamic shared-memory limit once per (kernel, device, size).
template <class K>
cudaError_t prepare(K kernel, int dyn, int static_bytes, int* done_per_device) {
  if (dyn + static_bytes <= 48 * 1024) return cudaSuccess;
  int devid = 0;
  cudaError_t e = cudaGetDevice(&devid);
  if (e != cudaSuccess) return e;
  if (devid >= 0 && devid < 64 && done_per_device[devid] >= dyn) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e != cudaSuccess) return e;
  if (devid >= 0 && devid < 64) done_per_device[devid] = dyn;
  return cudaSuccess;
}

int g_dequant_dyn[64];
int g_dequant_dyn16[64];

}  // namespace

cudaError_t launch_decode(const PoolDev& P, const int32_t* slots, int B, const float* q,
                          const float* k, const float* v, const float* gate,
                          const float* beta, float* out, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  if (P.scheme == SCHEME_ROW_ABSMAX) return launch_decode_absmax(P, slots, B, q, k, v, gate, beta, out, s);
  const unsigned n = unsigned(B) * unsigned(P.H);
  constexpr int SM = 2 * sizeof(DecodeSmem);
  if (P.scale16) {
    if (P.any_mixed) return launch_persistent<decode_kernel<StepQuantStore, true, true>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
    return launch_persistent<decode_kernel<StepQuantStore, false, true>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
  }
  if (P.any_mixed) return launch_persistent<decode_kernel<StepQuantStore, true, false>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
  return launch_persistent<decode_kernel<StepQuantStore, false, false>>(n, SM, s, P, slots, B, q, k, v, gate, beta, out);
}

cudaError_t launch_quantize(const PoolDev& P, const int32_t* slots, int B, const float* S,
                            cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  if (P.scheme == SCHEME_ROW_ABSMAX) return launch_quantize_absmax(P, slots, B, S, s);
  const unsigned n = unsigned(B) * unsigned(P.H);
  constexpr int SM = sizeof(CtaSmem);
  if (P.scale16) return launch_items<quantize_kernel<StepQuantStore, true>>(n, SM, s, P, slots, B, S);
  return launch_items<quantize_kernel<StepQuantStore, false>>(n, SM, s, P, slots, B, S);
}

cudaError_t launch_dequantize(const PoolDev& P, const int32_t* slots, int B, float* S_out,
                              cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const int dyn = stage_bytes(P);
  if (P.scale16) {
    cudaError_t e = prepare(dequant_kernel<true>, dyn, 2 * D * 4, g_dequant_dyn16);
    if (e != cudaSuccess) return e;
    dequant_kernel<true><<<B * P.H, NT, dyn, s>>>(P, slots, B, S_out);
  } else {
    cudaError_t e = prepare(dequant_kernel<false>, dyn, 2 * D * 4, g_dequant_dyn);
    if (e != cudaSuccess) return e;
    dequant_kernel<false><<<B * P.H, NT, dyn, s>>>(P, slots, B, S_out);
  }
  return cudaGetLastError();
}

cudaError_t launch_fp32_step(int kind, int B, int H, float* S, const float* q, const float* k,
                             const float* v, const float* gate, const float* beta, float* out,
                             cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  fp32_step_kernel<<<B * H, NT, 0, s>>>(kind, S, q, k, v, gate, beta, out);
  return cudaGetLastError();
}

}  // namespace stq
