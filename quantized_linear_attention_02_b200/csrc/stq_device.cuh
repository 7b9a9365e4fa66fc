// Device code shared by the kernels of the packed Delta-rule state step: code formats,
// per-warp staging, the restore / delta-update / readout part of the decode step and
// the kernel bodies. The quantiser that ends a decode step (and stq_quantize_init) is a
// policy `Store` with
//   template <int BITS> static __device__ void store(CtaSmem&, WarpRows&,
//       f2 (&s)[RPW][2], const Scales<H16>& sc, uint8_t* codes, int warp_code_start,
//       float* o, uint8_t* stage);
// which quantises the warp's 16 rows s (float32 state), writes codes and scales (r at
// Scales index i, c at D + j) and, when o is not null, the readout whose per-warp
// partials are in red[1][0]. `stage` is the warp's consumed code staging area (its
// rows' bytes), free for the store to use.
// The float32 evaluation order is described at the top of stq_kernels.cu.
#pragma once

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
// aligned row. kStaged: the row sits in a warp's shared-memory staging buffer (sized for
// 8-bit rows), so the word after a 6-bit row's last code may be read unconditionally.
template <int BITS, bool kStaged = false>
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
      // hi is used only when sh > 8, and then wi + 1 <= 23
      const uint32_t hi = (kStaged || sh > 8) ? wp[wi + 1] : 0u;
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

// The lane's codes u0..u3 (columns 4l..4l+3) clamped in two pairs of 16-bit lanes, u0 and
// u2 in one word and u1 and u3 in the other, so that w02 | w13 << b already holds u0 | u1 << b
// in its low half and u2 | u3 << b in its high half (2b <= 16).
__device__ __forceinline__ void clamp_pairs(f2 t01, f2 t23, uint32_t hi, uint32_t& w02, uint32_t& w13) {
  w02 = clamp_s16x2(__byte_perm(__float_as_uint(t01.x), __float_as_uint(t23.x), 0x5410), hi);
  w13 = clamp_s16x2(__byte_perm(__float_as_uint(t01.y), __float_as_uint(t23.y), 0x5410), hi);
}

template <int BITS>
__device__ __forceinline__ void store_codes_s16(uint8_t* row, int lane, f2 t01, f2 t23, uint32_t hi) {
  uint32_t w02, w13;
  clamp_pairs(t01, t23, hi, w02, w13);
  if constexpr (BITS == 8) {
    reinterpret_cast<uint32_t*>(row)[lane] = __byte_perm(w02, w13, 0x6240);
  } else {
    const uint32_t x = w02 + (w13 << BITS);     // u0 | u1 << b, u2 | u3 << b at bit 16
    if constexpr (BITS == 4) {
      reinterpret_cast<uint16_t*>(row)[lane] = static_cast<uint16_t>(__byte_perm(x, 0u, 0x0020));
    } else if constexpr (BITS == 2) {
      row[lane] = static_cast<uint8_t>(x | (x >> 12));
    } else {
      // the high half moves down to bit 12; bits 24.. are not stored
      const uint32_t f = (x & 0xFFFu) | ((x >> 4) & ~0xFFFu);
      // even lanes: 16 bits at byte 3l, 8 bits at 3l + 2; odd lanes: 8 bits at 3l, 16 at 3l + 1
      const int odd = lane & 1;
      uint8_t* p8 = row + 3 * lane + 2 - 2 * odd;
      uint16_t* p16 = reinterpret_cast<uint16_t*>(row + 3 * lane + odd);
      *p8 = static_cast<uint8_t>(f >> (16 - 16 * odd));
      *p16 = static_cast<uint16_t>(f >> (8 * odd));
    }
  }
}

// Copy `bytes` (multiple of 16) with 16-byte accesses by the whole CTA.
__device__ __forceinline__ void copy16(void* dst, const void* src, int bytes) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int t = threadIdx.x; t < (bytes >> 4); t += NT) d[t] = s[t];
}

// r[D] then c[D] of one head in its slot: float32, or binary16 (H16) in a compact pool.
template <bool H16>
struct Scales {
  void* p;
  __device__ __forceinline__ float get(int i) const {
    if constexpr (H16) return __half2float(static_cast<const __half*>(p)[i]);
    else return static_cast<const float*>(p)[i];
  }
  __device__ __forceinline__ float4 get4(int i) const {   // i a multiple of 4
    if constexpr (!H16) {
      return *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
    } else {
      const uint2 b = *reinterpret_cast<const uint2*>(static_cast<const __half*>(p) + i);
      return make_float4(__half2float(__ushort_as_half(uint16_t(b.x & 0xFFFFu))),
                         __half2float(__ushort_as_half(uint16_t(b.x >> 16))),
                         __half2float(__ushort_as_half(uint16_t(b.y & 0xFFFFu))),
                         __half2float(__ushort_as_half(uint16_t(b.y >> 16))));
    }
  }
  __device__ __forceinline__ void put(int i, float v) const {
    if constexpr (H16) static_cast<__half*>(p)[i] = __float2half_rn(v);
    else static_cast<float*>(p)[i] = v;
  }
  // the value the pool will hold: binary16 rounding (to nearest even) in a compact pool
  __device__ __forceinline__ float stored(float v) const {
    if constexpr (H16) return __half2float(__float2half_rn(v));
    else return v;
  }
};

template <bool H16>
struct HeadRef {
  uint8_t* codes;      // global: this head's codes in its slot
  uint16_t* pivots;    // global: this head's first pivot row in its slot
  Scales<H16> sc;      // global: r[D], c[D] of this head in its slot
  int code_bytes;
  int piv_count;
  int bits;            // uniform width of the head, 16 if all pivot, 0 if mixed
  int piv_stage_off;   // byte offset of the pivot rows in the staging buffer
  uint32_t* err;       // the pool's sticky error word (checked builds record into it)
};

template <bool H16>
__device__ __forceinline__ HeadRef<H16> head_ref(const PoolDev& P, int slot, int h) {
  HeadRef<H16> r;
  r.err = P.err;
  r.code_bytes = int(P.head_code_bytes[h]);
  r.piv_count = int(P.head_piv_count[h]);
  r.bits = int(P.head_bits[h]);
  r.codes = P.codes + uint64_t(slot) * P.slot_code_bytes + P.head_code_off[h];
  r.pivots = P.pivots + (uint64_t(slot) * P.n_pivot_rows + P.head_piv_first[h]) * D;
  r.sc.p = static_cast<uint8_t*>(P.scales) + (uint64_t(slot) * P.H + h) * 2 * D * (H16 ? 2 : 4);
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
  uint4 rk[RPW];                   // mixed heads, unpack of row i (width b, pivot rows 0):
                                   //   {M = 2^b - 1, M << b, exponent bits of a code at
                                   //   bit b, 4b | 2b << 8 | byte offset of the row in the
                                   //   warp's codes << 16}
  float4 rp[RPW];                  // restore of row i: -(2^23 + 2^(b-1)), -(2^(23-b) +
                                   //   2^(b-1)), dec_i r_i, 0 (pivot rows: 0, 0, dec_i r_i, 0)
  uint4 st[RPW];                   // final codes of row i: {bits of 1.5*2^23 + 2^(b-1),
                                   //   (2^b - 1) * 0x10001, 2^(2b) - 1,
                                   //   b | (16 - 2b) << 8 | row offset << 16}
                                   //   (pivot rows: {.., 0, 0, 16})
  f2 clampb[RPW];                  // least-squares clamp: 1.5*2^23 -+ qmax
  uint32_t info[RPW];              // bits | offset << 8
  uint8_t codes[2][RPW * D];       // this warp's rows of packed codes: the item being
                                   // decoded and the next one (arriving asynchronously)
  uint32_t tail[4];                // the last row may read one word past its codes
};

// The inputs of one (request, head) item that a warp needs, as they arrive from global
// memory by asynchronous copies issued while the warp works on the item before it.
struct __align__(16) WarpRaw {
  float k[RPW], q[RPW];            // k_i, q_i of rows 16w..16w+15
  float gate[RPW];                 // per-row retention (KDA)
  float v[RPW];                    // v_j of the columns 16w..16w+15 that lanes 0..15 own
  uint32_t info[RPW];              // row_info of the rows
  float g[RPW], om[RPW];           // row gain and omega of the rows
  uint32_t r[RPW];                 // r_i of the rows (float32; binary16 in the first 32 bytes)
  uint32_t c[D];                   // c_j (float32; binary16 in the first 256 bytes)
  float beta, gate_s;              // beta and the GDN retention of the item
  int32_t next_slot;               // slot of the warp's next item
  int32_t slot;                    // slot of this item
  uint4 next_rec;                  // warp_rec of the next item
  uint4 rec;                       // warp_rec of this item
};

struct __align__(16) CtaSmem {
  float4 red[2][2][NW][D / 4];     // ping-pong partials: [buffer][quantity][warp][col/4]
  float col_ic[D];                 // 1/c_j of the current column scale, from its owner
  float col_delta[D];              // delta_j = beta (v_j - u_j), from its owner
  WarpRows wr[NW];
};

struct __align__(16) DecodeSmem {
  CtaSmem cs;
  WarpRaw raw[NW];
  const uint8_t* ptab[8];          // base pointers of the prefetched row arrays
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// Store the low byte of v at shared-memory address `addr` where `pred` holds, as a
// predicated instruction (no branch).
__device__ __forceinline__ void st_shared_u8_if(bool pred, uint32_t addr, uint32_t v) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p st.shared.u8 [%0], %1;\n\t}"
               ::"r"(addr), "r"(v), "r"(int(pred))
               : "memory");
}

// Mixed-width rows: pack this lane's four codes of one row (t = 1.5*2^23 + bias + n in the
// low 16 bits, |n| < 2^15) with the row's store constants T (WarpRows::st), clamped to
// [1, 2^b - 1] in 16-bit lanes, and store its b/2 bytes into the warp's staging area at
// shared address `stage_s` (the area takes the pool's layout of the warp's rows). Any width
// runs the same instructions; a pivot row (zero constants) stores nothing.
__device__ __forceinline__ void stage_mixed_codes(uint4 T, f2 t01, f2 t23, uint32_t stage_s, int lane) {
  const int bits = int(T.w & 0xFFu);
  const bool code_row = bits != PIVOT;
  uint32_t w02, w13;
  clamp_pairs(t01, t23, T.y, w02, w13);
  // funnel shifts take their count mod 32: b and 16 - 2b straight from T.w
  const uint32_t x = w02 | __funnelshift_l(0u, w13, T.w);                // u0 | u1 << b, u2 | u3 << b at 16
  const uint32_t f = (x & T.z) | (__funnelshift_r(x, 0u, T.w >> 8) & ~T.z);
  const uint32_t dst = stage_s + (T.w >> 16) + uint32_t((bits * lane) >> 1);
  st_shared_u8_if(code_row, dst, f);
  st_shared_u8_if(code_row && bits >= 4, dst + 1, f >> 8);
  st_shared_u8_if(code_row && bits >= 6, dst + 2, f >> 16);
  st_shared_u8_if(code_row && bits >= 8, dst + 3, f >> 24);
}

// Copy the warp's staged codes (16 b bytes per quantised row, in the pool's layout) to the
// pool at `dst` with 16-byte stores.
__device__ __forceinline__ void copy_out_staged(const WarpRows& wr, const uint8_t* stage, uint8_t* dst, int lane) {
  const uint32_t my = lane < RPW ? (row_bits(wr.info[lane]) == PIVOT ? 0u : 16u * row_bits(wr.info[lane])) : 0u;
  const int bytes = int(__reduce_add_sync(0xffffffffu, my));
  __syncwarp();
  for (int o = 16 * lane; o < bytes; o += 16 * 32)
    *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(stage + o);
}

// The same copy issued only where `pred` holds, as a predicated instruction (no branch);
// where it does not, nothing is read or written.
__device__ __forceinline__ void cp_async16_if(bool pred, void* dst, const void* src) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}"
      ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src), "r"(int(pred))
      : "memory");
}

// The 256 threads (8 warps) that work on one (request, head) item meet at a named
// barrier of their own: 1 for threads 0..255, 2 for 256..511 (a decode CTA runs two such
// groups on separate items; a 256-thread CTA is one group).
__device__ __forceinline__ int group_id() { return int(threadIdx.x) >> 8; }
__device__ __forceinline__ int group_tid() { return int(threadIdx.x) & (NT - 1); }
__device__ __forceinline__ void group_sync() {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + group_id()) : "memory");
}
__device__ __forceinline__ int group_sync_or(int pred) {
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.s32 p, %1, 0;\n\tbar.red.or.pred q, %2, 256, p;\n\t"
      "selp.s32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred), "r"(1 + group_id())
      : "memory");
  return r;
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

// Lane l < 16 of a warp: every per-row constant of its row (width `bits`, codes at byte
// `code_off` of the warp's codes, decay times stored row scale `rd`) that the mixed-width
// paths read, packed per phase. A pivot row gets zero unpack and store constants and
// offset 0, so that it can run the code path harmlessly.
__device__ __forceinline__ void mixed_row_consts(WarpRows& wr, int l, int bits, uint32_t code_off, float rd) {
  float qm, iq, mb;
  width_consts(bits, qm, iq, mb);
  wr.qm[l] = qm; wr.iq[l] = iq; wr.mb[l] = mb;
  wr.clampb[l] = make_float2(MAGIC - qm, MAGIC + qm);
  if (bits == PIVOT) {
    wr.rk[l] = make_uint4(0u, 0u, 0u, 0u);
    wr.rp[l] = make_float4(0.0f, 0.0f, rd, 0.0f);
    wr.st[l] = make_uint4(__float_as_uint(mb), 0u, 0u, uint32_t(PIVOT));
  } else {
    const uint32_t M = (1u << bits) - 1u;
    const float bias = float(1 << (bits - 1));
    wr.rk[l] = make_uint4(M, M << bits, uint32_t(150 - bits) << 23,
                          uint32_t(4 * bits) | (uint32_t(2 * bits) << 8) | (code_off << 16));
    wr.rp[l] = make_float4(-(8388608.0f + bias), -(float(1u << (23 - bits)) + bias), rd, 0.0f);
    wr.st[l] = make_uint4(__float_as_uint(mb), M * 0x00010001u, (1u << (2 * bits)) - 1u,
                          uint32_t(bits) | (uint32_t(16 - 2 * bits) << 8) | (code_off << 16));
  }
}

// Lanes 0..15 of warp w: the per-row data of rows 16w..16w+15 of head h.
template <bool H16>
__device__ __forceinline__ void load_warp_rows(const PoolDev& P, int h, WarpRows& wr, int lane, int r0,
                                               const float* k_vec, const float* q_vec, const Scales<H16>* r_in,
                                               const float* gate_rows, float gate_s) {
  if (lane < RPW) {
    const int i = r0 + lane;
    const uint32_t info = P.row_info[h * D + i];
    wr.info[lane] = info;
    wr.g[lane] = P.g[h * D + i];
    wr.om[lane] = P.omega[h * D + i];
    mixed_row_consts(wr, lane, row_bits(info), uint32_t(row_off(info)) - P.warp_code_off[h * NW + r0 / RPW], 0.0f);
    if (k_vec != nullptr) {
      const float dec = gate_rows != nullptr ? gate_rows[i] : gate_s;
      const float kv = k_vec[i], qv = q_vec[i];
      const float rd = fmul(dec, r_in->get(i));
      wr.dec[lane] = dec;
      wr.kk[lane] = make_float2(kv, kv);
      wr.qq[lane] = make_float2(qv, qv);
      wr.rdd[lane] = make_float2(rd, rd);
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
  // lanes 16..31 repeat the work of lanes 0..15 (no divergent branch); only 0..15 store
  const int j = 16 * w + (lane & 15);
  const float* part = reinterpret_cast<const float*>(cs.red[0][0][0]);
  float x[NW];
#pragma unroll
  for (int ww = 0; ww < NW; ++ww) x[ww] = part[ww * D + j];
  const float u = fadd(fadd(fadd(x[0], x[1]), fadd(x[2], x[3])), fadd(fadd(x[4], x[5]), fadd(x[6], x[7])));
  const float dl = fmul(beta_s, fadd(v_own, -u));
  if (lane < 16) cs.col_delta[j] = dl;
}

template <int BITS, class Store, bool H16>
__device__ __forceinline__ void decode_warp(CtaSmem& cs, WarpRows& wr, const HeadRef<H16>& hr, int warp_code_start,
                                            uint8_t* wcodes, const f2 (&cin)[2], float v_own, float beta_s,
                                            float* o_out) {
  const int tid = group_tid(), w = tid >> 5, lane = tid & 31;
  f2 s[RPW][2];
#ifdef STQ_CHECKS
  bool zero_code = false;   // a stored code 0: never written by the quantiser
#endif

  // ---- restore S' = D (r c Q) and the column sums u_j = sum_i k_i S'_ij ---------------
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    if constexpr (BITS == MIXED) {
      // any width b: the lane's 4b bits start at bit 4 b l of the row (the word after them
      // is inside the staging area: the next row, the other buffer or `tail`); codes 0
      // and 2 sit at bit 0 of f and fh, codes 1 and 3 at bit b, each unpacked in place
      // into a float's mantissa (2^23 + u, 2^(23-b) + u). Every row runs this path: a
      // pivot row's zero constants and zero stored row scale make it 0 here, and the
      // fix-up after the loop replaces it.
      const uint4 K = wr.rk[rr];
      const float4 P4 = wr.rp[rr];
      const f2 off = make_float2(P4.x, P4.y);
      const uint32_t* wp = reinterpret_cast<const uint32_t*>(wcodes + (K.w >> 16));
      const int bitpos = int(K.w & 0xFFu) * lane;
      const uint32_t f = __funnelshift_r(wp[bitpos >> 5], wp[(bitpos >> 5) + 1], bitpos & 31);
      const uint32_t fh = f >> ((K.w >> 8) & 0xFFu);
#ifdef STQ_CHECKS
      zero_code |= row_bits(wr.info[rr]) != PIVOT &&
                   ((f & K.x) == 0 || (f & K.y) == 0 || (fh & K.x) == 0 || (fh & K.y) == 0);
#endif
      const f2 q01 = add2(make_float2(__uint_as_float((f & K.x) | FLOAT_2P23), __uint_as_float((f & K.y) | K.z)), off);
      const f2 q23 = add2(make_float2(__uint_as_float((fh & K.x) | FLOAT_2P23), __uint_as_float((fh & K.y) | K.z)), off);
      const f2 rd = dup(P4.z);
      s[rr][0] = mul2(mul2(q01, rd), cin[0]);
      s[rr][1] = mul2(mul2(q23, rd), cin[1]);
    } else {
      uint32_t cd[4];
      load_codes<BITS, true>(wcodes + rr * (D * BITS / 8), lane, cd);
#ifdef STQ_CHECKS
      // the mantissa of an unpacked code holds u << pos: zero exactly when u = 0
      zero_code |= ((cd[0] & 0x7FFFFFu) == 0) || ((cd[1] & 0x7FFFFFu) == 0) ||
                   ((cd[2] & 0x7FFFFFu) == 0) || ((cd[3] & 0x7FFFFFu) == 0);
#endif
      const float4 r2 = *reinterpret_cast<const float4*>(&wr.rdd[rr & ~1]);
      const f2 rd = (rr & 1) ? make_float2(r2.z, r2.w) : make_float2(r2.x, r2.y);
      f2 q01, q23;
      codes_to_q<BITS>(cd, q01, q23);
      s[rr][0] = mul2(mul2(q01, rd), cin[0]);
      s[rr][1] = mul2(mul2(q23, rd), cin[1]);
    }
  }
  if (BITS == MIXED && hr.piv_count) {
    // FP16 pivot rows: S' = D h
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const uint32_t info = wr.info[rr];
      if (row_bits(info) == PIVOT) {
        const uint2 hv = *reinterpret_cast<const uint2*>(hr.pivots + row_off(info) * D + 4 * lane);
        f2 x, y;
        half4_floats(hv, x, y);
        const f2 dd = dup(wr.dec[rr]);
        s[rr][0] = mul2(dd, x);
        s[rr][1] = mul2(dd, y);
      }
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
  group_sync();

  // ---- delta_j = beta (v_j - u_j) by its column owner; S = S' + k delta^T; readout ----
  f2 delta[2];
  publish_delta(cs, lane, w, v_own, beta_s);
  group_sync();
  {
    const float4 d4 = *reinterpret_cast<const float4*>(&cs.col_delta[4 * lane]);
    delta[0] = make_float2(d4.x, d4.y);
    delta[1] = make_float2(d4.z, d4.w);
  }
  {
    // S = S' + k delta^T and the readout partials sum_i q_i S_ij of this warp's rows (the
    // readout is compared within a tolerance, not bit for bit: plain running sums, even
    // and odd rows apart)
    f2 o[2][2] = {{make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)}, {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)}};
#pragma unroll
    for (int m = 0; m < RPW / 2; ++m) {
      const float4 k2 = *reinterpret_cast<const float4*>(&wr.kk[2 * m]);
      const float4 q2 = *reinterpret_cast<const float4*>(&wr.qq[2 * m]);
      const f2 kp[2] = {make_float2(k2.x, k2.y), make_float2(k2.z, k2.w)};
      const f2 qp[2] = {make_float2(q2.x, q2.y), make_float2(q2.z, q2.w)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        s[2 * m + e][0] = fma2(kp[e], delta[0], s[2 * m + e][0]);
        s[2 * m + e][1] = fma2(kp[e], delta[1], s[2 * m + e][1]);
        o[e][0] = fma2(qp[e], s[2 * m + e][0], o[e][0]);
        o[e][1] = fma2(qp[e], s[2 * m + e][1], o[e][1]);
      }
    }
    put_partial(cs.red[1][0], w, lane, add2(o[0][0], o[1][0]), add2(o[0][1], o[1][1]));
  }
  if (BITS == MIXED && hr.piv_count) {
    // pivot rows: store float16(S) now (they take no part in the refit)
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const uint32_t info = wr.info[rr];
      if (row_bits(info) == PIVOT)
        *reinterpret_cast<uint2*>(hr.pivots + row_off(info) * D + 4 * lane) = half4_bits(s[rr][0], s[rr][1]);
    }
  }
#ifdef STQ_CHECKS
  {
    bool nonfinite = false;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr)
      nonfinite |= !isfinite(s[rr][0].x) || !isfinite(s[rr][0].y) || !isfinite(s[rr][1].x) ||
                   !isfinite(s[rr][1].y);
    const uint32_t bits = (__any_sync(0xffffffffu, zero_code) ? ERR_CODE : 0u) |
                          (__any_sync(0xffffffffu, nonfinite) ? ERR_NONFINITE : 0u);
    if (lane == 0 && bits) atomicOr(hr.err, bits);
  }
#endif
  Store::template store<BITS>(cs, wr, s, hr.sc, hr.codes, warp_code_start, o_out, wcodes);
}

// A head whose rows are all FP16 pivots: decay, update, readout, store float16; r = c = 0.
template <bool H16>
__device__ __forceinline__ void decode_pivot_warp(CtaSmem& cs, WarpRows& wr, const HeadRef<H16>& hr,
                                                  float v_own, float beta_s, float* o_out) {
  const int tid = group_tid(), w = tid >> 5, lane = tid & 31;
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
  group_sync();
  f2 delta[2];
  publish_delta(cs, lane, w, v_own, beta_s);
  group_sync();
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
  group_sync();
  if (w == 0) {
    f2 lo, hi;
    warp_tree(cs.red[1][0], lane, lo, hi);
    *reinterpret_cast<float4*>(o_out + 4 * lane) = make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  if (tid < 2 * D) hr.sc.put(tid, 0.0f);
}

__device__ __forceinline__ void cp_async4_if(bool pred, void* dst, const void* src) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p cp.async.ca.shared.global [%0], [%1], 4;\n\t}"
      ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src), "r"(int(pred))
      : "memory");
}

// Warp w's asynchronous copies of the inputs of item (h, bq): its packed rows into
// `codes_dst`, its rows' k, q, gate, row data and r, the column scales c and the v_j of
// its owned columns into `raw`; and, when there is a following item (hn, bn), that
// item's slot and warp_rec. The slot and warp_rec of (h, bq) itself came from the
// previous copies and are stored into `raw` as they are. A slot outside [0, n_slots)
// gets no copies (the item is skipped and flagged when its turn comes).
// `ptab` holds the eight 64-byte row arrays' base pointers: k, q, gate, v, row_info, g,
// omega, scales.
template <bool H16>
__device__ __forceinline__ void prefetch_item(const PoolDev& P, const int32_t* __restrict__ slots,
                                              const float* __restrict__ beta, const float* __restrict__ gate,
                                              const uint8_t* const* ptab, WarpRaw& raw, uint8_t* codes_dst,
                                              int h, int bq, int slot, uint4 rec, bool has_next, int hn,
                                              int bn, int w, int lane) {
  constexpr int ES = H16 ? 2 : 4;   // bytes per stored scale
  const int r0 = w * RPW;
  if (lane == 0) {
    raw.slot = slot;
    raw.rec = rec;
  }
  // every copy is predicated (no branch); the addresses of a skipped item or of a
  // missing next item are formed from index 0 and never used
  const bool ok = slot >= 0 && slot < P.n_slots;
  const int sl = ok ? slot : 0;
  const uint64_t vi = uint64_t(bq) * P.H + h;
  const uint64_t soff = (uint64_t(sl) * P.H + h) * (2 * D * ES);
  const uint8_t* cg = P.codes + uint64_t(sl) * P.slot_code_bytes + rec.x + rec.y;
#pragma unroll
  for (int j = 0; j < (RPW * D) / (16 * 32); ++j) {
    const int o = 16 * lane + 16 * 32 * j;
    cp_async16_if(ok && o < int(rec.z), codes_dst + o, cg + o);
  }
  // eight 64-byte row arrays, four lanes each; v of the 16 columns the warp owns shares
  // the rows' offset (r0 = 16 w)
  const int grp = lane >> 2, part = 16 * (lane & 3);
  const uint64_t off = grp < 4 ? (vi * D + r0) * 4 : grp < 7 ? (uint64_t(h) * D + r0) * 4 : soff + r0 * ES;
  const bool valid = (grp != 2 || P.kind != 0) && (grp != 7 || part < RPW * ES);
  cp_async16_if(ok && valid, reinterpret_cast<uint8_t*>(&raw) + 64 * grp + part, ptab[grp] + off + part);
  cp_async16_if(ok && 16 * lane < D * ES, reinterpret_cast<uint8_t*>(raw.c) + 16 * lane,
                ptab[7] + soff + D * ES + 16 * lane);
  cp_async4_if(ok && lane == 4, &raw.beta, beta + vi);
  cp_async4_if(ok && lane == 5 && P.kind == 0, &raw.gate_s, gate + vi);
  const int nb = has_next ? bn : 0, nh = has_next ? hn : 0;
  cp_async4_if(has_next && lane == 6, &raw.next_slot, slots + nb);
  cp_async16_if(has_next && lane == 7, &raw.next_rec, P.warp_rec + nh * NW + w);
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// ---------------------------------------------------------------------------------
// stq_decode_step: persistent CTAs, each taking the (head, request) items
// blockIdx.x, blockIdx.x + gridDim.x, ... of a head-major numbering (the CTAs resident
// on an SM at the same time mostly run the same width's code path). Each warp copies
// the inputs of its next item into shared memory asynchronously while it decodes the
// current one, so no global load is waited for inside the loop; it writes its own
// codes back, so the CTA synchronises only for the column exchanges.
// ---------------------------------------------------------------------------------
template <class Store, bool kMixed, bool H16>
__global__ void __launch_bounds__(2 * NT, 1)
decode_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, const float* __restrict__ q,
              const float* __restrict__ k, const float* __restrict__ v,
              const float* __restrict__ gate, const float* __restrict__ beta,
              float* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_bytes[];
  const int grp = group_id();
  DecodeSmem& sm = reinterpret_cast<DecodeSmem*>(smem_bytes)[grp];
  CtaSmem& cs = sm.cs;
  const int tid = group_tid(), w = tid >> 5, lane = tid & 31;
  WarpRows& wr = cs.wr[w];
  WarpRaw& raw = sm.raw[w];
  if (tid < 8) {
    const void* base = tid == 0 ? static_cast<const void*>(k) : tid == 1 ? static_cast<const void*>(q)
                     : tid == 2 ? static_cast<const void*>(gate) : tid == 3 ? static_cast<const void*>(v)
                     : tid == 4 ? static_cast<const void*>(P.row_info) : tid == 5 ? static_cast<const void*>(P.g)
                     : tid == 6 ? static_cast<const void*>(P.omega) : static_cast<const void*>(P.scales);
    sm.ptab[tid] = static_cast<const uint8_t*>(base);
  }
  group_sync();
  // group g of CTA b takes the items m = 2 b + g, 2 b + g + 2 gridDim.x, ..., with
  // m = h * B + bq; the next one is reached by adding (dh, db) with one carry (no
  // division inside the loop)
  const int G = 2 * int(gridDim.x);
  const int dh = G / B, db = G - dh * B;
  const int m0 = 2 * int(blockIdx.x) + grp;
  int h = m0 / B, bq = m0 - h * B;
  if (h >= P.H) return;
  // the second group starts about half an item later, so that the two groups sharing
  // the SM are mostly in different phases of the step (a bounded, one-time wait)
  if (grp == 1)
    for (int i = 0; i < 8; ++i) __nanosleep(500);
  {
    int hn = h + dh, bn = bq + db;
    if (bn >= B) { bn -= B; ++hn; }
    prefetch_item<H16>(P, slots, beta, gate, sm.ptab, raw, wr.codes[0], h, bq, slots[bq],
                       P.warp_rec[h * NW + w], hn < P.H, hn, bn, w, lane);
  }
  for (int cur = 0; h < P.H; cur ^= 1) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
    const int slot = raw.slot;
    const uint4 rec = raw.rec;
    // this item's row data -> the working area (lanes 0..15, one row each)
    if (lane < RPW) {
      const uint32_t info = raw.info[lane];
      wr.info[lane] = info;
      wr.g[lane] = raw.g[lane];
      wr.om[lane] = raw.om[lane];
      const float dec = (P.kind == 0) ? raw.gate_s : raw.gate[lane];
      float r_in;
      if constexpr (H16) r_in = __half2float(reinterpret_cast<const __half*>(raw.r)[lane]);
      else r_in = __uint_as_float(raw.r[lane]);
      const float rd = fmul(dec, r_in);
      if constexpr (kMixed) mixed_row_consts(wr, lane, row_bits(info), uint32_t(row_off(info)) - rec.y, rd);
      const float kv = raw.k[lane], qv = raw.q[lane];
      wr.dec[lane] = dec;
      wr.kk[lane] = make_float2(kv, kv);
      wr.qq[lane] = make_float2(qv, qv);
      wr.rdd[lane] = make_float2(rd, rd);
    }
    const float beta_s = raw.beta;
    f2 cin[2];
    if constexpr (H16) {
      const uint2 hb = reinterpret_cast<const uint2*>(raw.c)[lane];
      half4_floats(hb, cin[0], cin[1]);
    } else {
      const float4 c4 = reinterpret_cast<const float4*>(raw.c)[lane];
      cin[0] = make_float2(c4.x, c4.y);
      cin[1] = make_float2(c4.z, c4.w);
    }
    const float v_own = raw.v[lane & 15];
    // this warp's pivot rows (warp-uniform): mixed-width warps without any skip the fix-ups
    const int npiv = __popc(__ballot_sync(0xffffffffu, lane < RPW && row_bits(raw.info[lane]) == PIVOT));
    int hn = h + dh, bn = bq + db;
    if (bn >= B) { bn -= B; ++hn; }
    if (hn < P.H) {
      const int next_slot = raw.next_slot;
      const uint4 next_rec = raw.next_rec;
      int hnn = hn + dh, bnn = bn + db;
      if (bnn >= B) { bnn -= B; ++hnn; }
      __syncwarp();   // the raw area is consumed: the next item's copies may overwrite it
      prefetch_item<H16>(P, slots, beta, gate, sm.ptab, raw, wr.codes[cur ^ 1], hn, bn, next_slot, next_rec,
                         hnn < P.H, hnn, bnn, w, lane);
    }
    if (slot >= 0 && slot < P.n_slots) {
      HeadRef<H16> hr;
      hr.err = P.err;
      hr.codes = P.codes + uint64_t(slot) * P.slot_code_bytes + rec.x;
      hr.pivots = P.pivots + (uint64_t(slot) * P.n_pivot_rows + (rec.w >> 8)) * D;
      hr.sc.p = static_cast<uint8_t*>(P.scales) + (uint64_t(slot) * P.H + h) * 2 * D * (H16 ? 2 : 4);
      hr.bits = int(rec.w & 0xFFu);
      hr.code_bytes = 0;     // not used by the decode step
      hr.piv_count = npiv;   // pivot rows among this warp's rows
      hr.piv_stage_off = 0;
      const int wstart = int(rec.y);
      uint8_t* wcodes = wr.codes[cur];
      float* o_out = out + (uint64_t(bq) * P.H + h) * D;
      switch (hr.bits) {
        case 2: decode_warp<2, Store, H16>(cs, wr, hr, wstart, wcodes, cin, v_own, beta_s, o_out); break;
        case 4: decode_warp<4, Store, H16>(cs, wr, hr, wstart, wcodes, cin, v_own, beta_s, o_out); break;
        case 6: decode_warp<6, Store, H16>(cs, wr, hr, wstart, wcodes, cin, v_own, beta_s, o_out); break;
        case 8: decode_warp<8, Store, H16>(cs, wr, hr, wstart, wcodes, cin, v_own, beta_s, o_out); break;
        case PIVOT: decode_pivot_warp(cs, wr, hr, v_own, beta_s, o_out); break;
        default:
          // heads whose rows have different widths (only pools with such heads launch this)
          if constexpr (kMixed) decode_warp<MIXED, Store, H16>(cs, wr, hr, wstart, wcodes, cin, v_own, beta_s, o_out);
          break;
      }
    } else if (tid == 0) {
      atomicOr(P.err, ERR_SLOT_RANGE);
    }
    h = hn;
    bq = bn;
  }
}

// ---------------------------------------------------------------------------------
// stq_quantize_init: float32 states -> packed pool.
// ---------------------------------------------------------------------------------
template <int BITS, class Store, bool H16>
__device__ __forceinline__ void quantize_warp(CtaSmem& cs, WarpRows& wr, const HeadRef<H16>& hr, int warp_code_start,
                                              const float* src) {
  const int tid = group_tid(), w = tid >> 5, lane = tid & 31;
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
  Store::template store<BITS>(cs, wr, s, hr.sc, hr.codes, warp_code_start, nullptr, wr.codes[0]);
}

template <class Store, bool H16>
__global__ void __launch_bounds__(NT, 2)
quantize_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, const float* __restrict__ S) {
  extern __shared__ __align__(16) uint8_t smem_bytes[];
  CtaSmem& cs = *reinterpret_cast<CtaSmem*>(smem_bytes);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int r0 = w * RPW;
  const int item = blockIdx.x;
  const int bq = item / P.H, h = item - bq * P.H;
  const int slot = slots[bq];
  if (slot < 0 || slot >= P.n_slots) {
    if (tid == 0) atomicOr(P.err, ERR_SLOT_RANGE);
    return;
  }
  const HeadRef<H16> hr = head_ref<H16>(P, slot, h);
  WarpRows& wr = cs.wr[w];
  load_warp_rows<H16>(P, h, wr, lane, r0, nullptr, nullptr, nullptr, nullptr, 0.0f);
  __syncwarp();
  const int wstart = int(P.warp_code_off[h * NW + w]);
  const float* src = S + uint64_t(item) * D * D;
  switch (hr.bits) {
    case 2: quantize_warp<2, Store, H16>(cs, wr, hr, wstart, src); break;
    case 4: quantize_warp<4, Store, H16>(cs, wr, hr, wstart, src); break;
    case 6: quantize_warp<6, Store, H16>(cs, wr, hr, wstart, src); break;
    case 8: quantize_warp<8, Store, H16>(cs, wr, hr, wstart, src); break;
    case PIVOT:
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const int i = r0 + rr;
        const float4 x = *reinterpret_cast<const float4*>(src + i * D + 4 * lane);
        *reinterpret_cast<uint2*>(hr.pivots + i * D + 4 * lane) =
            half4_bits(make_float2(x.x, x.y), make_float2(x.z, x.w));
      }
      if (tid < 2 * D) hr.sc.put(tid, 0.0f);
      break;
    default: quantize_warp<MIXED, Store, H16>(cs, wr, hr, wstart, src); break;
  }
}

// ---------------------------------------------------------------------------------
// Launch helpers. Kernels whose shared memory exceeds the default 48 KB raise their
// limit once per device; the persistent decode kernel runs as many CTAs as fit on the
// device at once (SM count x resident CTAs per SM, also found once per device).
// ---------------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

template <auto Kern>
cudaError_t kernel_setup(int smem, int* per_device_cap, int threads = NT) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static int cap_cache[kMaxDevices];
  int cap = (dev >= 0 && dev < kMaxDevices) ? cap_cache[dev] : 0;
  if (cap == 0) {
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int nsm = 0, per = 0;
    e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, Kern, threads, smem);
    if (e != cudaSuccess) return e;
    cap = nsm * (per > 0 ? per : 1);
    if (dev >= 0 && dev < kMaxDevices) cap_cache[dev] = cap;
  }
  *per_device_cap = cap;
  return cudaSuccess;
}

// One CTA per item (grid = n_items), dynamic shared memory `smem`.
template <auto Kern, class... Args>
cudaError_t launch_items(unsigned n_items, int smem, cudaStream_t s, Args... args) {
  int cap = 0;
  cudaError_t e = kernel_setup<Kern>(smem, &cap);
  if (e != cudaSuccess) return e;
  Kern<<<n_items, NT, smem, s>>>(args...);
  return cudaGetLastError();
}

// Persistent decode CTAs of two 256-thread groups, each on its own items: grid =
// min(ceil(n_items / 2), CTAs resident on the device at once).
template <auto Kern, class... Args>
cudaError_t launch_persistent(unsigned n_items, int smem, cudaStream_t s, Args... args) {
  int cap = 0;
  cudaError_t e = kernel_setup<Kern>(smem, &cap, 2 * NT);
  if (e != cudaSuccess) return e;
  const unsigned pairs = (n_items + 1) / 2;
  const unsigned grid = pairs < unsigned(cap) ? pairs : unsigned(cap);
  Kern<<<grid, 2 * NT, smem, s>>>(args...);
  return cudaGetLastError();
}

}  // namespace
}  // namespace stq
