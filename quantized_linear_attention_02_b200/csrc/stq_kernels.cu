// Kernels of the packed Delta-rule state decode step for B200 (sm_100a).
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
// Quantization" (arXiv 2609.38169) as its web pages describe it -- gated delta rule
// (bloombook.cn tutorial, section 2), readout before requantisation (singularity-lens
// summary, decode-order paragraph), dual-axis scales r_i c_j z_ij (bloombook section 4),
// per-unit widths and FP16 pivot units (ai-trend review, Method).
//
// One CTA of 256 threads owns one (request, head) 128x128 state. Warp w holds key rows
// 16w..16w+15, lane l holds value columns 4l..4l+3 as two float2 pairs, so a thread keeps
// 64 state values in registers for the whole step. A row's width is uniform across a
// warp instruction (KDA widths vary per key row without divergence); heads whose rows
// share one width run a code path specialised for it.
//
// Float32 evaluation order (the CPU oracle restates the same order):
//   * sums over the 128 rows of a column or the 128 columns of a row are balanced
//     binary trees, adjacent pairs first. Column sums: a thread's 16 rows form the
//     lower 4 levels, the 8 warps (shared memory) the top 3. Row sums: a thread's 4
//     columns form the lower 2 levels, butterfly shuffle steps xor 1,2,...,16 the top 5;
//   * in a sum of products a_i b_i each adjacent pair is one fused multiply-add,
//     fma(a_2m, b_2m, a_2m+1 * b_2m+1); the state update is S = fma(k, delta, S'); every
//     other product is rounded on its own (explicit _rn forms, --fmad=false);
//   * the quantiser's x = y * inv_c is taken exactly: fma(y, inv_c, 1.5*2^23) rounds the
//     exact product to the nearest integer (ties to even) inside the 2^23 binade, and
//     clamping is done in that binade, where the low bits are the (biased) code.
#include <cuda_fp16.h>

#include "stq_internal.h"

namespace stq {
namespace {

constexpr int NT = 256;   // threads per head-state
constexpr int NW = 8;     // warps per head-state
constexpr int RPW = 16;   // key rows per warp
constexpr float MAGIC = 12582912.0f;        // 1.5 * 2^23
constexpr uint32_t FLOAT_2P23 = 0x4B000000u;
constexpr float SMALLEST_NORMAL = 1.17549435e-38f;  // 2^-126
constexpr int MIXED = 0;

using f2 = float2;

__device__ __forceinline__ float fmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float fadd(float a, float b) { return __fadd_rn(a, b); }
// Packed float2 arithmetic (one rounding per component, like the scalar _rn forms). The
// code generator fuses a multiply that feeds an add, so every sum of products below is
// written with explicit fused pairs and leaves no multiply-add pair to fuse.
__device__ __forceinline__ f2 mul2(f2 a, f2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ f2 add2(f2 a, f2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ f2 dup(float x) { return make_float2(x, x); }

// 1/a correctly rounded for a >= 2^-126; 0 for a smaller (or zero) scale.
__device__ __forceinline__ float recip_scale(float a) {
  return a >= SMALLEST_NORMAL ? __frcp_rn(a) : 0.0f;
}

template <int N>
struct V2 {
  f2 x[N];
};

// Balanced binary tree over leaves f(LO), ..., f(LO+N-1), each a V2<M> of independent
// column sums.
template <int LO, int N, int M, class F>
__device__ __forceinline__ V2<M> tree(F&& f) {
  if constexpr (N == 1) {
    return f(LO);
  } else {
    V2<M> a = tree<LO, N / 2, M>(f);
    V2<M> b = tree<LO + N / 2, N / 2, M>(f);
#pragma unroll
    for (int m = 0; m < M; ++m) a.x[m] = add2(a.x[m], b.x[m]);
    return a;
  }
}

__device__ __forceinline__ int row_bits(uint32_t info) { return int(info & 0xFFu); }
__device__ __forceinline__ int row_off(uint32_t info) { return int(info >> 8); }

// ---------------------------------------------------------------------------------
// code formats: code j of a b-bit row is bits [b*j, b*j+b) of a little-endian stream;
// lane l owns codes 4l..4l+3 = bits [4bl, 4bl+4b) = bytes [bl/2, bl/2 + b/2)
// ---------------------------------------------------------------------------------

// Bit position the unpacked code k of a lane sits at inside its float's mantissa. The
// float is 2^(23 - pos) + u exactly (exponent 127 + 23 - pos, u * 2^pos in the mantissa,
// which needs u * 2^pos < 2^23), so no code has to be shifted down to bit 0.
template <int BITS>
__host__ __device__ constexpr int code_pos(int k) {
  return BITS == 8 ? 0 : BITS == 6 ? (k == 3 ? 17 : 6 * k) : BITS * k;
}
template <int BITS>
__host__ __device__ constexpr uint32_t code_exp(int k) {
  return uint32_t(127 + 23 - code_pos<BITS>(k)) << 23;
}
// 2^(23 - pos) + bias: subtracting it from the unpacked float gives Q = u - bias exactly.
template <int BITS>
__host__ __device__ constexpr float code_offset(int k) {
  return float(1u << (23 - code_pos<BITS>(k))) + float(1 << (BITS - 1));
}

// The four codes of a lane as floats 2^(23 - pos_k) + u_k (exact), from a 16-byte
// aligned row.
template <int BITS>
__device__ __forceinline__ void load_codes(const uint8_t* row, int lane, uint32_t (&c)[4]) {
  if constexpr (BITS == 8) {
    const uint32_t w = reinterpret_cast<const uint32_t*>(row)[lane];
    c[0] = __byte_perm(w, FLOAT_2P23, 0x7540);
    c[1] = __byte_perm(w, FLOAT_2P23, 0x7541);
    c[2] = __byte_perm(w, FLOAT_2P23, 0x7542);
    c[3] = __byte_perm(w, FLOAT_2P23, 0x7543);
  } else {
    constexpr uint32_t M = (1u << BITS) - 1u;
    uint32_t f, f3;
    if constexpr (BITS == 4) {
      f = reinterpret_cast<const uint16_t*>(row)[lane];
      f3 = f;
    } else if constexpr (BITS == 2) {
      f = row[lane];
      f3 = f;
    } else {
      // 6 bits: bytes 3l..3l+2, inside word 3l/4 and possibly the next one; code 3 is
      // taken one bit lower (position 17) from a second funnel shift
      const uint32_t* wp = reinterpret_cast<const uint32_t*>(row);
      const int byte = 3 * lane, wi = byte >> 2, sh = (byte & 3) * 8;
      const uint32_t lo = wp[wi];
      const uint32_t hi = (sh > 8) ? wp[wi + 1] : 0u;  // wi + 1 <= 23 whenever sh > 8
      f = __funnelshift_r(lo, hi, sh);
      f3 = __funnelshift_r(lo, hi, sh + 1);
    }
    c[0] = (f & (M << code_pos<BITS>(0))) | code_exp<BITS>(0);
    c[1] = (f & (M << code_pos<BITS>(1))) | code_exp<BITS>(1);
    c[2] = (f & (M << code_pos<BITS>(2))) | code_exp<BITS>(2);
    c[3] = (f3 & (M << code_pos<BITS>(3))) | code_exp<BITS>(3);
  }
}

// Q of the four codes as two float pairs.
template <int BITS>
__device__ __forceinline__ void codes_to_q(const uint32_t (&cd)[4], f2& q01, f2& q23) {
  q01 = add2(make_float2(__uint_as_float(cd[0]), __uint_as_float(cd[1])),
             make_float2(-code_offset<BITS>(0), -code_offset<BITS>(1)));
  q23 = add2(make_float2(__uint_as_float(cd[2]), __uint_as_float(cd[3])),
             make_float2(-code_offset<BITS>(2), -code_offset<BITS>(3)));
}

// Pack four biased codes (low bits of t = 1.5*2^23 + u) and store them into a row.
template <int BITS>
__device__ __forceinline__ void store_codes(uint8_t* row, int lane, const uint32_t (&t)[4]) {
  if constexpr (BITS == 8) {
    const uint32_t p01 = __byte_perm(t[0], t[1], 0x0040);
    const uint32_t p23 = __byte_perm(t[2], t[3], 0x0040);
    reinterpret_cast<uint32_t*>(row)[lane] = __byte_perm(p01, p23, 0x5410);
  } else {
    constexpr uint32_t M = (1u << BITS) - 1u;
    const uint32_t f = (t[0] & M) | ((t[1] & M) << BITS) | ((t[2] & M) << (2 * BITS)) |
                       ((t[3] & M) << (3 * BITS));
    if constexpr (BITS == 4) {
      reinterpret_cast<uint16_t*>(row)[lane] = static_cast<uint16_t>(f);
    } else if constexpr (BITS == 2) {
      row[lane] = static_cast<uint8_t>(f);
    } else {
      // 24 bits at byte 3l: one 16-bit and one 8-bit store, the 16-bit one aligned
      const bool odd = lane & 1;
      uint8_t* p = row + 3 * lane;
      uint8_t* p8 = odd ? p : p + 2;
      uint16_t* p16 = reinterpret_cast<uint16_t*>(odd ? p + 1 : p);
      *p8 = static_cast<uint8_t>(odd ? f : (f >> 16));
      *p16 = static_cast<uint16_t>(odd ? (f >> 8) : f);
    }
  }
}

// Final codes in 16-bit lanes. t = fma(y, 1/c, 1.5*2^23 + bias) holds bias + n in its low
// 16 bits (two's complement) whenever |n| < 2^15, n = rint(y / c); two such low halves
// are clamped to [1, 2^b - 1] = bias + [-qmax, qmax] with one packed min and one packed
// max, then packed. The caller guarantees |n| < 2^15 (see refit_store).
__device__ __forceinline__ uint32_t clamp_s16x2(uint32_t x, uint32_t hi) {
  uint32_t y;
  asm("max.s16x2 %0, %1, %2;" : "=r"(y) : "r"(x), "r"(0x00010001u));
  asm("min.s16x2 %0, %1, %2;" : "=r"(y) : "r"(y), "r"(hi));
  return y;
}

template <int BITS>
__device__ __forceinline__ void store_codes_s16(uint8_t* row, int lane, f2 t01, f2 t23, uint32_t hi) {
  const uint32_t w01 = clamp_s16x2(__byte_perm(__float_as_uint(t01.x), __float_as_uint(t01.y), 0x5410), hi);
  const uint32_t w23 = clamp_s16x2(__byte_perm(__float_as_uint(t23.x), __float_as_uint(t23.y), 0x5410), hi);
  if constexpr (BITS == 8) {
    reinterpret_cast<uint32_t*>(row)[lane] = __byte_perm(w01, w23, 0x6420);
  } else if constexpr (BITS == 4) {
    const uint32_t x01 = w01 | (w01 >> 12), x23 = w23 | (w23 >> 12);
    reinterpret_cast<uint16_t*>(row)[lane] = static_cast<uint16_t>(__byte_perm(x01, x23, 0x0040));
  } else if constexpr (BITS == 2) {
    const uint32_t x = w01 | (w23 << 4);
    row[lane] = static_cast<uint8_t>(x | (x >> 14));
  } else {
    const uint32_t x01 = w01 | (w01 >> 10), x23 = w23 | (w23 >> 10);
    const uint32_t f = (x01 & 0xFFFu) | (x23 << 12);   // bits 24.. are not stored
    const bool odd = lane & 1;
    uint8_t* p = row + 3 * lane;
    uint8_t* p8 = odd ? p : p + 2;
    uint16_t* p16 = reinterpret_cast<uint16_t*>(odd ? p + 1 : p);
    *p8 = static_cast<uint8_t>(odd ? f : (f >> 16));
    *p16 = static_cast<uint16_t>(odd ? (f >> 8) : f);
  }
}

// Copy `bytes` (multiple of 16) with 16-byte accesses by the whole CTA.
__device__ __forceinline__ void copy16(void* dst, const void* src, int bytes) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int t = threadIdx.x; t < (bytes >> 4); t += NT) d[t] = s[t];
}

struct HeadRef {
  uint8_t* codes;      // global: this head's codes in its slot
  uint16_t* pivots;    // global: this head's first pivot row in its slot
  float* scales;       // global: r[D], c[D] of this head in its slot
  int code_bytes;
  int piv_count;
  int bits;            // uniform width of the head, 16 if all pivot, 0 if mixed
  int piv_stage_off;   // byte offset of the pivot rows in the staging buffer
};

__device__ __forceinline__ HeadRef head_ref(const PoolDev& P, int slot, int h) {
  HeadRef r;
  r.code_bytes = int(P.head_code_bytes[h]);
  r.piv_count = int(P.head_piv_count[h]);
  r.bits = int(P.head_bits[h]);
  r.codes = P.codes + uint64_t(slot) * P.slot_code_bytes + P.head_code_off[h];
  r.pivots = P.pivots + (uint64_t(slot) * P.n_pivot_rows + P.head_piv_first[h]) * D;
  r.scales = P.scales + (uint64_t(slot) * P.H + h) * 2 * D;
  r.piv_stage_off = r.code_bytes;  // code bytes are a multiple of 16
  return r;
}

__device__ __forceinline__ uint2 half4_bits(f2 a, f2 b) {
  const uint32_t lo = uint32_t(__half_as_ushort(__float2half_rn(a.x))) |
                      (uint32_t(__half_as_ushort(__float2half_rn(a.y))) << 16);
  const uint32_t hi = uint32_t(__half_as_ushort(__float2half_rn(b.x))) |
                      (uint32_t(__half_as_ushort(__float2half_rn(b.y))) << 16);
  return make_uint2(lo, hi);
}

__device__ __forceinline__ void half4_floats(uint2 hv, f2& a, f2& b) {
  a.x = __half2float(__ushort_as_half(uint16_t(hv.x & 0xFFFFu)));
  a.y = __half2float(__ushort_as_half(uint16_t(hv.x >> 16)));
  b.x = __half2float(__ushort_as_half(uint16_t(hv.y & 0xFFFFu)));
  b.y = __half2float(__ushort_as_half(uint16_t(hv.y >> 16)));
}

// Sum of the 8 warps' partials of one quantity for this lane's 4 columns, as a tree
// ((w0+w1)+(w2+w3))+((w4+w5)+(w6+w7)).
__device__ __forceinline__ void warp_tree(const float4 (*red)[D / 4], int lane, f2& lo, f2& hi) {
  f2 a[NW], b[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const float4 v = red[w][lane];
    a[w] = make_float2(v.x, v.y);
    b[w] = make_float2(v.z, v.w);
  }
  lo = add2(add2(add2(a[0], a[1]), add2(a[2], a[3])), add2(add2(a[4], a[5]), add2(a[6], a[7])));
  hi = add2(add2(add2(b[0], b[1]), add2(b[2], b[3])), add2(add2(b[4], b[5]), add2(b[6], b[7])));
}

__device__ __forceinline__ void put_partial(float4 (*red)[D / 4], int w, int lane, f2 lo, f2 hi) {
  red[w][lane] = make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Restore one row of S' = D (r c Q) for this lane's 4 columns.
template <int BITS>
__device__ __forceinline__ void restore_row(const uint8_t* row, int lane, float rd,
                                            const f2 (&cin)[2], f2& s01, f2& s23) {
  uint32_t cd[4];
  load_codes<BITS>(row, lane, cd);
  f2 q01, q23;
  codes_to_q<BITS>(cd, q01, q23);
  s01 = mul2(mul2(q01, dup(rd)), cin[0]);
  s23 = mul2(mul2(q23, dup(rd)), cin[1]);
}

// ---------------------------------------------------------------------------------
// Shared memory. Each warp stages and uses only its own 16 key rows (WarpRows), so the
// only CTA-wide synchronisation is the exchange of column partial sums (red).
// ---------------------------------------------------------------------------------
struct __align__(16) WarpRows {
  f2 kk[RPW], qq[RPW], rdd[RPW];   // (k_i, k_i), (q_i, q_i), (dec_i r_i, dec_i r_i)
  f2 irr[RPW], bb[RPW];            // refit: (1/r_i, 1/r_i), (omega_i r_i^2, same)
  float dec[RPW];                  // row retention
  float g[RPW], om[RPW];           // row gain and omega
  float qm[RPW], iq[RPW], mb[RPW];   // per-row width constants (mixed heads)
  uint32_t info[RPW];              // bits | offset << 8
  uint8_t codes[RPW * D];          // this warp's rows of packed codes
};

struct __align__(16) CtaSmem {
  float4 red[2][2][NW][D / 4];     // ping-pong partials: [buffer][quantity][warp][col/4]
  float col_ic[D];                 // 1/c_j of the current column scale, from its owner
  float col_delta[D];              // delta_j = beta (v_j - u_j), from its owner
  WarpRows wr[NW];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// Per-row constants of a width (2/4/6/8, 16 = pivot).
__device__ __forceinline__ void width_consts(int bits, float& qm, float& iq, float& mb) {
  if (bits == PIVOT) {
    qm = 0.0f; iq = 0.0f; mb = MAGIC;
  } else {
    const int bias = 1 << (bits - 1);
    qm = float(bias - 1);
    iq = __frcp_rn(qm);
    mb = MAGIC + float(bias);
  }
}

// Lanes 0..15 of warp w: the per-row data of rows 16w..16w+15 of head h.
__device__ __forceinline__ void load_warp_rows(const PoolDev& P, int h, WarpRows& wr, int lane, int r0,
                                               const float* k_vec, const float* q_vec, const float* r_in,
                                               const float* gate_rows, float gate_s) {
  if (lane < RPW) {
    const int i = r0 + lane;
    const uint32_t info = P.row_info[h * D + i];
    wr.info[lane] = info;
    wr.g[lane] = P.g[h * D + i];
    wr.om[lane] = P.omega[h * D + i];
    float qm, iq, mb;
    width_consts(row_bits(info), qm, iq, mb);
    wr.qm[lane] = qm; wr.iq[lane] = iq; wr.mb[lane] = mb;
    if (k_vec != nullptr) {
      const float dec = gate_rows != nullptr ? gate_rows[i] : gate_s;
      const float kv = k_vec[i], qv = q_vec[i];
      const float rd = fmul(dec, r_in[i]);
      wr.dec[lane] = dec;
      wr.kk[lane] = make_float2(kv, kv);
      wr.qq[lane] = make_float2(qv, qv);
      wr.rdd[lane] = make_float2(rd, rd);
    }
  }
}

// ---------------------------------------------------------------------------------
// Refit of this warp's rows: row scale, column scale start, two omega-weighted
// least-squares steps, final codes (bloombook section 4; singularity-lens dual-axis
// paragraph). On entry s[][] holds the float32 state (pivot rows already stored) and the
// caller may have put readout partials into red[1][0]. The codes go straight to the
// pool; r of this warp's rows is written; c (this lane's columns) is returned.
// Four CTA barriers: column maximum, step one, step two (and the caller's u exchange).
// ---------------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ void refit_store(CtaSmem& cs, WarpRows& wr, f2 (&s)[RPW][2], float* r_global,
                                            float* c_global, uint8_t* codes_global, int warp_code_start,
                                            float* o_global) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = w * RPW;

  // --- row scale r_i = (tree sum_j |S_ij|) / 128 * g_i -------------------------------
  float a[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr)
    a[rr] = fadd(fadd(fabsf(s[rr][0].x), fabsf(s[rr][0].y)), fadd(fabsf(s[rr][1].x), fabsf(s[rr][1].y)));
  // reduce-scatter over lanes: step m keeps half of the rows and pairs lane l with l^m
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const bool up = lane & 1;
    const float send = up ? a[t] : a[t + 8];
    const float keep = up ? a[t + 8] : a[t];
    a[t] = fadd(keep, __shfl_xor_sync(0xffffffffu, send, 1));
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const bool up = lane & 2;
    const float send = up ? a[t] : a[t + 4];
    const float keep = up ? a[t + 4] : a[t];
    a[t] = fadd(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const bool up = lane & 4;
    const float send = up ? a[t] : a[t + 2];
    const float keep = up ? a[t + 2] : a[t];
    a[t] = fadd(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
  {
    const bool up = lane & 8;
    const float send = up ? a[0] : a[1];
    const float keep = up ? a[1] : a[0];
    a[0] = fadd(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
  a[0] = fadd(a[0], __shfl_xor_sync(0xffffffffu, a[0], 16));
  {
    // lane l now holds the sum of row R(l): bits 0..3 of l chose halves 8, 4, 2, 1
    const int R = ((lane & 1) << 3) | ((lane & 2) << 1) | ((lane & 4) >> 1) | ((lane & 8) >> 3);
    const bool pivot = (BITS == MIXED) ? (row_bits(wr.info[R]) == PIVOT) : false;
    const float r = pivot ? 0.0f : fmul(fmul(a[0], 0.0078125f), wr.g[R]);
    if (lane < 16) {
      const float ir = recip_scale(r), bv = fmul(wr.om[R], fmul(r, r));
      wr.irr[R] = make_float2(ir, ir);
      wr.bb[R] = make_float2(bv, bv);
      r_global[r0 + R] = r;
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
      const float iq = wr.iq[rr];
      mx[0] = fmaxf(mx[0], fmul(fabsf(s[rr][0].x), iq));
      mx[1] = fmaxf(mx[1], fmul(fabsf(s[rr][0].y), iq));
      mx[2] = fmaxf(mx[2], fmul(fabsf(s[rr][1].x), iq));
      mx[3] = fmaxf(mx[3], fmul(fabsf(s[rr][1].y), iq));
    } else {
      mx[0] = fmaxf(mx[0], fabsf(s[rr][0].x));
      mx[1] = fmaxf(mx[1], fabsf(s[rr][0].y));
      mx[2] = fmaxf(mx[2], fabsf(s[rr][1].x));
      mx[3] = fmaxf(mx[3], fabsf(s[rr][1].y));
    }
  }
  cs.red[1][1][w][lane] = make_float4(mx[0], mx[1], mx[2], mx[3]);
  __syncthreads();

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
    if (lane < 16) cs.col_ic[jown] = recip_scale(c_own);
  }
  const float c0 = c_own;
  int wide = 0, any_wide = 0;
  __syncthreads();

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
          lo_b = MAGIC - wr.qm[rr];
          hi_b = MAGIC + wr.qm[rr];
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
    __syncthreads();
    {
      // lanes 0..15: numerator of column jown, lanes 16..31: its denominator
      const float* part = reinterpret_cast<const float*>(cs.red[it][lane >> 4][0]);
      float x[NW];
#pragma unroll
      for (int ww = 0; ww < NW; ++ww) x[ww] = part[ww * D + jown];
      const float sum = fadd(fadd(fadd(x[0], x[1]), fadd(x[2], x[3])), fadd(fadd(x[4], x[5]), fadd(x[6], x[7])));
      const float den = __shfl_down_sync(0xffffffffu, sum, 16);
      if (lane < 16) {
        if (den > 0.0f) c_own = __fdiv_rn(sum, den);
        const float icn = recip_scale(c_own);
        cs.col_ic[jown] = icn;
        // every least-squares step keeps c >= c_before / 2 (each term Q y >= c Q^2 / 2),
        // so |n| = |rint(y / c)| <= qmax c0 / c + 1/2 < 2^15 unless rounding at the bottom
        // of the float32 range broke that; then the column takes the float clamp
        if (BITS != MIXED && it == 1) wide = !(fmul(c0, icn) < 128.0f);
      }
    }
    if (BITS != MIXED && it == 1) any_wide = __syncthreads_or(wide);
    else __syncthreads();
  }

  // --- final codes with the final c, stored straight into the pool -------------------
  f2 ic[2];
  {
    const float4 i4 = *reinterpret_cast<const float4*>(&cs.col_ic[4 * lane]);
    ic[0] = make_float2(i4.x, i4.y);
    ic[1] = make_float2(i4.z, i4.w);
  }
  if (lane < 16) c_global[jown] = c_own;
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

// ---------------------------------------------------------------------------------
// One (request, head) of stq_decode_step, from this warp's staged rows.
// ---------------------------------------------------------------------------------
// Lane l < 16 of warp w owns column j = 16w + l: it sums the eight warps' partials of
// u_j = (k^T S')_j in the tree ((w0+w1)+(w2+w3))+((w4+w5)+(w6+w7)) and publishes
// delta_j = beta (v_j - u_j) through shared memory.
__device__ __forceinline__ void publish_delta(CtaSmem& cs, int lane, int w, float v_own, float beta_s) {
  if (lane < 16) {
    const int j = 16 * w + lane;
    const float* part = reinterpret_cast<const float*>(cs.red[0][0][0]);
    float x[NW];
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) x[ww] = part[ww * D + j];
    const float u = fadd(fadd(fadd(x[0], x[1]), fadd(x[2], x[3])), fadd(fadd(x[4], x[5]), fadd(x[6], x[7])));
    cs.col_delta[j] = fmul(beta_s, fadd(v_own, -u));
  }
}

template <int BITS>
__device__ __forceinline__ void decode_warp(CtaSmem& cs, WarpRows& wr, const HeadRef& hr, int warp_code_start,
                                            const f2 (&cin)[2], float v_own, float beta_s,
                                            float* o_out) {
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  f2 s[RPW][2];

  // ---- restore S' = D (r c Q) and the column sums u_j = sum_i k_i S'_ij ---------------
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    if constexpr (BITS == MIXED) {
      const uint32_t info = wr.info[rr];
      const int bits = row_bits(info);
      const uint8_t* row = wr.codes + (row_off(info) - warp_code_start);
      const float rd = wr.rdd[rr].x;
      switch (bits) {
        case 2: restore_row<2>(row, lane, rd, cin, s[rr][0], s[rr][1]); break;
        case 4: restore_row<4>(row, lane, rd, cin, s[rr][0], s[rr][1]); break;
        case 6: restore_row<6>(row, lane, rd, cin, s[rr][0], s[rr][1]); break;
        case 8: restore_row<8>(row, lane, rd, cin, s[rr][0], s[rr][1]); break;
        default: {
          const uint2 hv = *reinterpret_cast<const uint2*>(hr.pivots + row_off(info) * D + 4 * lane);
          f2 x, y;
          half4_floats(hv, x, y);
          const f2 dd = dup(wr.dec[rr]);
          s[rr][0] = mul2(dd, x);
          s[rr][1] = mul2(dd, y);
        }
      }
    } else {
      uint32_t cd[4];
      load_codes<BITS>(wr.codes + rr * (D * BITS / 8), lane, cd);
      const float4 r2 = *reinterpret_cast<const float4*>(&wr.rdd[rr & ~1]);
      const f2 rd = (rr & 1) ? make_float2(r2.z, r2.w) : make_float2(r2.x, r2.y);
      f2 q01, q23;
      codes_to_q<BITS>(cd, q01, q23);
      s[rr][0] = mul2(mul2(q01, rd), cin[0]);
      s[rr][1] = mul2(mul2(q23, rd), cin[1]);
    }
  }
  {
    V2<2> u = tree<0, RPW / 2, 2>([&](int m) {
      const float4 k2 = *reinterpret_cast<const float4*>(&wr.kk[2 * m]);
      const f2 ke = make_float2(k2.x, k2.y), ko = make_float2(k2.z, k2.w);
      V2<2> leaf;
      leaf.x[0] = fma2(ke, s[2 * m][0], mul2(ko, s[2 * m + 1][0]));
      leaf.x[1] = fma2(ke, s[2 * m][1], mul2(ko, s[2 * m + 1][1]));
      return leaf;
    });
    put_partial(cs.red[0][0], w, lane, u.x[0], u.x[1]);
  }
  __syncthreads();

  // ---- delta_j = beta (v_j - u_j) by its column owner; S = S' + k delta^T; readout ----
  f2 delta[2];
  publish_delta(cs, lane, w, v_own, beta_s);
  __syncthreads();
  {
    const float4 d4 = *reinterpret_cast<const float4*>(&cs.col_delta[4 * lane]);
    delta[0] = make_float2(d4.x, d4.y);
    delta[1] = make_float2(d4.z, d4.w);
  }
  {
    V2<2> o = tree<0, RPW / 2, 2>([&](int m) {
      const float4 k2 = *reinterpret_cast<const float4*>(&wr.kk[2 * m]);
      const float4 q2 = *reinterpret_cast<const float4*>(&wr.qq[2 * m]);
      const f2 kp[2] = {make_float2(k2.x, k2.y), make_float2(k2.z, k2.w)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[2 * m + e][0] = fma2(kp[e], delta[0], s[2 * m + e][0]);
        s[2 * m + e][1] = fma2(kp[e], delta[1], s[2 * m + e][1]);
      }
      const f2 qe = make_float2(q2.x, q2.y), qo = make_float2(q2.z, q2.w);
      V2<2> leaf;
      leaf.x[0] = fma2(qe, s[2 * m][0], mul2(qo, s[2 * m + 1][0]));
      leaf.x[1] = fma2(qe, s[2 * m][1], mul2(qo, s[2 * m + 1][1]));
      return leaf;
    });
    put_partial(cs.red[1][0], w, lane, o.x[0], o.x[1]);
  }
  if constexpr (BITS == MIXED) {
    // pivot rows: store float16(S) now (they take no part in the refit)
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const uint32_t info = wr.info[rr];
      if (row_bits(info) == PIVOT)
        *reinterpret_cast<uint2*>(hr.pivots + row_off(info) * D + 4 * lane) = half4_bits(s[rr][0], s[rr][1]);
    }
  }
  refit_store<BITS>(cs, wr, s, hr.scales, hr.scales + D, hr.codes, warp_code_start, o_out);
}

// A head whose rows are all FP16 pivots: decay, update, readout, store float16; r = c = 0.
__device__ __forceinline__ void decode_pivot_warp(CtaSmem& cs, WarpRows& wr, const HeadRef& hr,
                                                  float v_own, float beta_s, float* o_out) {
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int r0 = w * RPW;
  f2 s[RPW][2];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const uint2 hv = *reinterpret_cast<const uint2*>(hr.pivots + (r0 + rr) * D + 4 * lane);
    f2 x, y;
    half4_floats(hv, x, y);
    const f2 dd = dup(wr.dec[rr]);
    s[rr][0] = mul2(dd, x);
    s[rr][1] = mul2(dd, y);
  }
  {
    V2<2> u = tree<0, RPW / 2, 2>([&](int m) {
      const float4 k2 = *reinterpret_cast<const float4*>(&wr.kk[2 * m]);
      const f2 ke = make_float2(k2.x, k2.y), ko = make_float2(k2.z, k2.w);
      V2<2> leaf;
      leaf.x[0] = fma2(ke, s[2 * m][0], mul2(ko, s[2 * m + 1][0]));
      leaf.x[1] = fma2(ke, s[2 * m][1], mul2(ko, s[2 * m + 1][1]));
      return leaf;
    });
    put_partial(cs.red[0][0], w, lane, u.x[0], u.x[1]);
  }
  __syncthreads();
  f2 delta[2];
  publish_delta(cs, lane, w, v_own, beta_s);
  __syncthreads();
  {
    const float4 d4 = *reinterpret_cast<const float4*>(&cs.col_delta[4 * lane]);
    delta[0] = make_float2(d4.x, d4.y);
    delta[1] = make_float2(d4.z, d4.w);
  }
  V2<2> o = tree<0, RPW / 2, 2>([&](int m) {
    const float4 k2 = *reinterpret_cast<const float4*>(&wr.kk[2 * m]);
    const float4 q2 = *reinterpret_cast<const float4*>(&wr.qq[2 * m]);
    const f2 kp[2] = {make_float2(k2.x, k2.y), make_float2(k2.z, k2.w)};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      s[2 * m + e][0] = fma2(kp[e], delta[0], s[2 * m + e][0]);
      s[2 * m + e][1] = fma2(kp[e], delta[1], s[2 * m + e][1]);
    }
    const f2 qe = make_float2(q2.x, q2.y), qo = make_float2(q2.z, q2.w);
    V2<2> leaf;
    leaf.x[0] = fma2(qe, s[2 * m][0], mul2(qo, s[2 * m + 1][0]));
    leaf.x[1] = fma2(qe, s[2 * m][1], mul2(qo, s[2 * m + 1][1]));
    return leaf;
  });
  put_partial(cs.red[1][0], w, lane, o.x[0], o.x[1]);
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr)
    *reinterpret_cast<uint2*>(hr.pivots + (r0 + rr) * D + 4 * lane) = half4_bits(s[rr][0], s[rr][1]);
  __syncthreads();
  if (w == 0) {
    f2 lo, hi;
    warp_tree(cs.red[1][0], lane, lo, hi);
    *reinterpret_cast<float4*>(o_out + 4 * lane) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  if (tid < 2 * D) hr.scales[tid] = 0.0f;
}

// ---------------------------------------------------------------------------------
// stq_decode_step: one CTA per (head, request) item, numbered head-major so that the
// CTAs resident on an SM at the same time mostly run the same width's code path. Each
// warp stages its own 16 rows (asynchronous 16-byte copies) and writes its own codes
// back, so the CTA synchronises only for the five column exchanges.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 2)
decode_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, const float* __restrict__ q,
              const float* __restrict__ k, const float* __restrict__ v,
              const float* __restrict__ gate, const float* __restrict__ beta,
              float* __restrict__ out) {
  __shared__ CtaSmem cs;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int r0 = w * RPW;
  const int h = blockIdx.x / B, bq = blockIdx.x - h * B;
  const int slot = slots[bq];
  if (slot < 0 || slot >= P.n_slots) {
    if (tid == 0) atomicOr(P.err, ERR_SLOT_RANGE);
    return;
  }
  const HeadRef hr = head_ref(P, slot, h);
  const int vi = bq * P.H + h;
  const uint64_t vec = uint64_t(vi) * D;
  WarpRows& wr = cs.wr[w];
  // this warp's packed rows -> shared memory (16-byte asynchronous copies)
  const int wstart = int(P.warp_code_off[h * NW + w]);
  const int wend = (w + 1 < NW) ? int(P.warp_code_off[h * NW + w + 1]) : hr.code_bytes;
  for (int o = 16 * lane; o < wend - wstart; o += 16 * 32) cp_async16(wr.codes + o, hr.codes + wstart + o);
  asm volatile("cp.async.commit_group;" ::: "memory");
  const float gate_s = (P.kind == 0) ? gate[vi] : 0.0f;
  load_warp_rows(P, h, wr, lane, r0, k + vec, q + vec, hr.scales, P.kind == 0 ? nullptr : gate + vec, gate_s);
  const float beta_s = beta[vi];
  const float4 c4 = *reinterpret_cast<const float4*>(hr.scales + D + 4 * lane);
  const f2 cin[2] = {make_float2(c4.x, c4.y), make_float2(c4.z, c4.w)};
  const float v_own = v[vec + 16 * w + (lane & 15)];
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncwarp();
  float* o_out = out + vec;
  switch (hr.bits) {
    case 2: decode_warp<2>(cs, wr, hr, wstart, cin, v_own, beta_s, o_out); break;
    case 4: decode_warp<4>(cs, wr, hr, wstart, cin, v_own, beta_s, o_out); break;
    case 6: decode_warp<6>(cs, wr, hr, wstart, cin, v_own, beta_s, o_out); break;
    case 8: decode_warp<8>(cs, wr, hr, wstart, cin, v_own, beta_s, o_out); break;
    case PIVOT: decode_pivot_warp(cs, wr, hr, v_own, beta_s, o_out); break;
    default: decode_warp<MIXED>(cs, wr, hr, wstart, cin, v_own, beta_s, o_out); break;
  }
}

// ---------------------------------------------------------------------------------
// stq_quantize_init: float32 states -> packed pool.
// ---------------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ void quantize_warp(CtaSmem& cs, WarpRows& wr, const HeadRef& hr, int warp_code_start,
                                              const float* src) {
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int r0 = w * RPW;
  f2 s[RPW][2];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const float4 x = *reinterpret_cast<const float4*>(src + (r0 + rr) * D + 4 * lane);
    s[rr][0] = make_float2(x.x, x.y);
    s[rr][1] = make_float2(x.z, x.w);
    if constexpr (BITS == MIXED) {
      const uint32_t info = wr.info[rr];
      if (row_bits(info) == PIVOT)
        *reinterpret_cast<uint2*>(hr.pivots + row_off(info) * D + 4 * lane) = half4_bits(s[rr][0], s[rr][1]);
    }
  }
  refit_store<BITS>(cs, wr, s, hr.scales, hr.scales + D, hr.codes, warp_code_start, nullptr);
}

__global__ void __launch_bounds__(NT, 2)
quantize_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, const float* __restrict__ S) {
  __shared__ CtaSmem cs;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int r0 = w * RPW;
  const int item = blockIdx.x;
  const int bq = item / P.H, h = item - bq * P.H;
  const int slot = slots[bq];
  if (slot < 0 || slot >= P.n_slots) {
    if (tid == 0) atomicOr(P.err, ERR_SLOT_RANGE);
    return;
  }
  const HeadRef hr = head_ref(P, slot, h);
  WarpRows& wr = cs.wr[w];
  load_warp_rows(P, h, wr, lane, r0, nullptr, nullptr, nullptr, nullptr, 0.0f);
  __syncwarp();
  const int wstart = int(P.warp_code_off[h * NW + w]);
  const float* src = S + uint64_t(item) * D * D;
  switch (hr.bits) {
    case 2: quantize_warp<2>(cs, wr, hr, wstart, src); break;
    case 4: quantize_warp<4>(cs, wr, hr, wstart, src); break;
    case 6: quantize_warp<6>(cs, wr, hr, wstart, src); break;
    case 8: quantize_warp<8>(cs, wr, hr, wstart, src); break;
    case PIVOT:
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const int i = r0 + rr;
        const float4 x = *reinterpret_cast<const float4*>(src + i * D + 4 * lane);
        *reinterpret_cast<uint2*>(hr.pivots + i * D + 4 * lane) =
            half4_bits(make_float2(x.x, x.y), make_float2(x.z, x.w));
      }
      if (tid < 2 * D) hr.scales[tid] = 0.0f;
      break;
    default: quantize_warp<MIXED>(cs, wr, hr, wstart, src); break;
  }
}

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
  const HeadRef hr = head_ref(P, slot, h);
  if (tid < D) {
    info_s[tid] = P.row_info[h * D + tid];
    r_s[tid] = hr.scales[tid];
  }
  copy16(stage, hr.codes, hr.code_bytes);
  copy16(stage + hr.piv_stage_off, hr.pivots, hr.piv_count * D * 2);
  const float4 c4 = *reinterpret_cast<const float4*>(hr.scales + D + 4 * lane);
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

}  // namespace

cudaError_t launch_decode(const PoolDev& P, const int32_t* slots, int B, const float* q,
                          const float* k, const float* v, const float* gate,
                          const float* beta, float* out, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  decode_kernel<<<B * P.H, NT, 0, s>>>(P, slots, B, q, k, v, gate, beta, out);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const PoolDev& P, const int32_t* slots, int B, const float* S,
                            cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  quantize_kernel<<<B * P.H, NT, 0, s>>>(P, slots, B, S);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const PoolDev& P, const int32_t* slots, int B, float* S_out,
                              cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const int dyn = stage_bytes(P);
  cudaError_t e = prepare(dequant_kernel, dyn, 2 * D * 4, g_dequant_dyn);
  if (e != cudaSuccess) return e;
  dequant_kernel<<<B * P.H, NT, dyn, s>>>(P, slots, B, S_out);
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
