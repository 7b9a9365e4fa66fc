// Kernels of the packed Delta-rule state decode step for B200 (sm_100a).
//
// Method: "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
// Quantization" (arXiv 2609.38169) as its web pages describe it -- gated delta rule
// (bloombook.cn tutorial, section 2), readout before requantisation (singularity-lens
// summary, decode-order paragraph), dual-axis scales r_i c_j z_ij (bloombook section 4),
// per-unit widths and FP16 pivot units (ai-trend review, Method).
//
// One CTA of 256 threads owns one (request, head) 128x128 state. Warp w holds key rows
// 16w..16w+15, lane l holds value columns 4l..4l+3, so a thread keeps 64 state values
// in registers for the whole step. A row's width is therefore uniform across a warp
// instruction (KDA widths vary per key row without divergence).
//
// Float32 evaluation order (the CPU oracle restates the same order):
//   * every product is rounded before it is added (explicit __fmul_rn/__fadd_rn; the
//     file is also built with --fmad=false);
//   * sums over the 128 rows of a column or the 128 columns of a row are balanced
//     binary trees: adjacent pairs first. Column sums: a thread's 16 rows form the
//     lower 4 levels, the 8 warps (smem) the top 3. Row sums: a thread's 4 columns form
//     the lower 2 levels, 5 butterfly shuffle steps (xor 1,2,...,16) the top 5;
//   * the quantiser's x = y * inv_c is taken exactly: fma(y, inv_c, 1.5*2^23) rounds the
//     exact product to the nearest integer (ties to even) inside the 2^23 binade, and
//     clamping is done in that same binade.
#include <cuda_fp16.h>

#include "stq_internal.h"

namespace stq {
namespace {

constexpr int NT = 256;   // threads per head-state
constexpr int NW = 8;     // warps per head-state
constexpr int RPW = 16;   // key rows per warp
constexpr float MAGIC = 12582912.0f;        // 1.5 * 2^23
constexpr float TWO23 = 8388608.0f;         // 2^23
constexpr float SMALLEST_NORMAL = 1.17549435e-38f;  // 2^-126

__device__ __forceinline__ float fmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float fadd(float a, float b) { return __fadd_rn(a, b); }

// 1/a correctly rounded for a >= 2^-126; 0 for a smaller (or zero) scale.
__device__ __forceinline__ float recip_scale(float a) {
  return a >= SMALLEST_NORMAL ? __frcp_rn(a) : 0.0f;
}

template <int N>
struct Vec {
  float x[N];
};

// Balanced binary tree over leaves f(LO), ..., f(LO+N-1); each leaf is a Vec<M> of
// independent sums (one per value column held by the thread).
template <int LO, int N, int M, class F>
__device__ __forceinline__ Vec<M> tree(F&& f) {
  if constexpr (N == 1) {
    return f(LO);
  } else {
    Vec<M> a = tree<LO, N / 2, M>(f);
    Vec<M> b = tree<LO + N / 2, N / 2, M>(f);
#pragma unroll
    for (int m = 0; m < M; ++m) a.x[m] = fadd(a.x[m], b.x[m]);
    return a;
  }
}

struct __align__(16) HeadSmem {
  float k[D], q[D], v[D], dec[D];
  float rd[D];       // decayed input row scale dec_i * r_i
  float inv_r[D];    // 1/r_i of the refit
  float b[D];        // omega_i * r_i^2
  float qm[D];       // qmax_i (0 for pivot rows)
  float inv_qm[D];   // 1/qmax_i (0 for pivot rows)
  float mb[D];       // 1.5*2^23 + 2^(b-1): magic that yields the biased code
  uint32_t info[D];  // bits | offset << 8
  float red[2][2][NW][D];  // ping-pong partial sums: [buffer][quantity][warp][column]
  float beta;
};

__device__ __forceinline__ int row_bits(uint32_t info) { return int(info & 0xFFu); }
__device__ __forceinline__ int row_off(uint32_t info) { return int(info >> 8); }

// The 4*bits-bit field holding codes 4*lane .. 4*lane+3 of one row: code j of a b-bit
// row is bits [b*j, b*j+b) of a little-endian bit stream. `row` is 16-byte aligned.
__device__ __forceinline__ uint32_t lane_field(const uint8_t* row, int bits, int lane) {
  if (bits == 8) return reinterpret_cast<const uint32_t*>(row)[lane];
  if (bits == 4) return reinterpret_cast<const uint16_t*>(row)[lane];
  if (bits == 2) return row[lane];
  // 6 bits: bytes 3*lane .. 3*lane+2, within word 3*lane/4 and possibly the next one
  const uint32_t* wp = reinterpret_cast<const uint32_t*>(row);
  const int byte = 3 * lane, wi = byte >> 2, sh = (byte & 3) * 8;
  const uint32_t lo = wp[wi];
  const uint32_t hi = (sh > 8) ? wp[wi + 1] : 0u;  // wi + 1 <= 23 whenever sh > 8
  return __funnelshift_r(lo, hi, sh) & 0xFFFFFFu;
}

__device__ __forceinline__ void store_field(uint8_t* row, int bits, int lane, uint32_t f) {
  if (bits == 8) {
    reinterpret_cast<uint32_t*>(row)[lane] = f;
  } else if (bits == 4) {
    reinterpret_cast<uint16_t*>(row)[lane] = static_cast<uint16_t>(f);
  } else if (bits == 2) {
    row[lane] = static_cast<uint8_t>(f);
  } else {
    uint8_t* p = row + 3 * lane;
    p[0] = static_cast<uint8_t>(f);
    p[1] = static_cast<uint8_t>(f >> 8);
    p[2] = static_cast<uint8_t>(f >> 16);
  }
}

// Code u (< 2^22) minus its bias, as an exact float: (2^23 + u) - (2^23 + bias).
__device__ __forceinline__ float code_value(uint32_t u, float two23_plus_bias) {
  return __fsub_rn(__uint_as_float(u | 0x4B000000u), two23_plus_bias);
}

// Copy `bytes` (multiple of 16) from global to shared with 16-byte accesses.
__device__ __forceinline__ void copy16(void* dst, const void* src, int bytes) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int t = threadIdx.x; t < (bytes >> 4); t += NT) d[t] = s[t];
}

__device__ __forceinline__ void copy16_out(void* dst, const void* src, int bytes) {
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
  int piv_stage_off;   // byte offset of the pivot rows in the staging buffer
};

__device__ __forceinline__ HeadRef head_ref(const PoolDev& P, int slot, int h) {
  HeadRef r;
  r.code_bytes = int(P.head_code_bytes[h]);
  r.piv_count = int(P.head_piv_count[h]);
  r.codes = P.codes + uint64_t(slot) * P.slot_code_bytes + P.head_code_off[h];
  r.pivots = P.pivots + (uint64_t(slot) * P.n_pivot_rows + P.head_piv_first[h]) * D;
  r.scales = P.scales + (uint64_t(slot) * P.H + h) * 2 * D;
  r.piv_stage_off = r.code_bytes;  // code bytes are a multiple of 16
  return r;
}

// Per-row static data of head h into shared memory (threads 0..127, one row each).
__device__ __forceinline__ void load_row_meta(const PoolDev& P, int h, HeadSmem& sm) {
  const int i = threadIdx.x;
  if (i < D) {
    const uint32_t info = P.row_info[h * D + i];
    const int bits = row_bits(info);
    sm.info[i] = info;
    if (bits == PIVOT) {
      sm.qm[i] = 0.0f;
      sm.inv_qm[i] = 0.0f;
      sm.mb[i] = MAGIC;
    } else {
      const int bias = 1 << (bits - 1);
      sm.qm[i] = float(bias - 1);
      sm.inv_qm[i] = __frcp_rn(float(bias - 1));
      sm.mb[i] = MAGIC + float(bias);
    }
  }
}

// ---------------------------------------------------------------------------------
// Refit: row scale, column scale start, two omega-weighted least-squares steps, final
// codes (bloombook section 4; singularity-lens dual-axis paragraph). On entry the
// thread's 64 values s[][] hold the float32 state (pivot rows already stored) and the
// caller may have put readout partials into red[1][0]. On exit the packed codes of the
// head are in `stage`, r has been written to global, and c is returned in c_out.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void refit_pack(const PoolDev& P, int h, HeadSmem& sm, uint8_t* stage,
                                           float (&s)[RPW][4], float* r_global,
                                           float (&c_out)[4], float* o_global) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // --- row scale r_i = (tree sum_j |S_ij|) / 128 * g_i -------------------------------
  float a[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr)
    a[rr] = fadd(fadd(fabsf(s[rr][0]), fabsf(s[rr][1])), fadd(fabsf(s[rr][2]), fabsf(s[rr][3])));
  // reduce-scatter over lanes: step m keeps half of the rows, pairs lane l with l^m
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
    // lane l now holds the full sum of row R(l): bits 0..3 of l select halves 8,4,2,1
    const int R = ((lane & 1) << 3) | ((lane & 2) << 1) | ((lane & 4) >> 1) | ((lane & 8) >> 3);
    const int i = w * RPW + R;
    const bool pivot = row_bits(sm.info[i]) == PIVOT;
    const float g = P.g[h * D + i];
    const float om = P.omega[h * D + i];
    const float r = pivot ? 0.0f : fmul(fmul(a[0], 0.0078125f), g);
    if (lane < 16) {
      sm.inv_r[i] = recip_scale(r);
      sm.b[i] = fmul(om, fmul(r, r));
      r_global[i] = r;
    }
  }
  __syncwarp();

  // --- y = S * inv_r; column start c0_j = max_i |y_ij| / qmax_i -----------------------
  float mx[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const float ir = sm.inv_r[i], iq = sm.inv_qm[i];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      s[rr][cc] = fmul(s[rr][cc], ir);
      mx[cc] = fmaxf(mx[cc], fmul(fabsf(s[rr][cc]), iq));
    }
  }
  *reinterpret_cast<float4*>(&sm.red[1][1][w][4 * lane]) = make_float4(mx[0], mx[1], mx[2], mx[3]);
  __syncthreads();

  if (o_global != nullptr && w == 0) {
    float o[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int j = 4 * lane + cc;
      o[cc] = fadd(fadd(fadd(sm.red[1][0][0][j], sm.red[1][0][1][j]), fadd(sm.red[1][0][2][j], sm.red[1][0][3][j])),
                   fadd(fadd(sm.red[1][0][4][j], sm.red[1][0][5][j]), fadd(sm.red[1][0][6][j], sm.red[1][0][7][j])));
    }
    *reinterpret_cast<float4*>(o_global + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
  }
  float c[4];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    float m = 0.0f;
#pragma unroll
    for (int ww = 0; ww < NW; ++ww) m = fmaxf(m, sm.red[1][1][ww][4 * lane + cc]);
    c[cc] = m;
  }

  // --- two least-squares steps: c_j <- sum_i p y / sum_i p Q, p = b_i Q_ij -------------
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    float ic[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) ic[cc] = recip_scale(c[cc]);
    Vec<8> nd = tree<0, RPW, 8>([&](int rr) {
      const int i = w * RPW + rr;
      const float bi = sm.b[i], q = sm.qm[i];
      Vec<8> leaf;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float t = __fmaf_rn(s[rr][cc], ic[cc], MAGIC);
        if (it > 0) t = fminf(fmaxf(t, MAGIC - q), MAGIC + q);  // step one never clips
        const float Q = __fsub_rn(t, MAGIC);
        const float p = fmul(bi, Q);
        leaf.x[cc] = fmul(p, s[rr][cc]);
        leaf.x[4 + cc] = fmul(p, Q);
      }
      return leaf;
    });
    float(*buf)[NW][D] = sm.red[it];
    *reinterpret_cast<float4*>(&buf[0][w][4 * lane]) = make_float4(nd.x[0], nd.x[1], nd.x[2], nd.x[3]);
    *reinterpret_cast<float4*>(&buf[1][w][4 * lane]) = make_float4(nd.x[4], nd.x[5], nd.x[6], nd.x[7]);
    __syncthreads();
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int j = 4 * lane + cc;
      const float num = fadd(fadd(fadd(buf[0][0][j], buf[0][1][j]), fadd(buf[0][2][j], buf[0][3][j])),
                             fadd(fadd(buf[0][4][j], buf[0][5][j]), fadd(buf[0][6][j], buf[0][7][j])));
      const float den = fadd(fadd(fadd(buf[1][0][j], buf[1][1][j]), fadd(buf[1][2][j], buf[1][3][j])),
                             fadd(fadd(buf[1][4][j], buf[1][5][j]), fadd(buf[1][6][j], buf[1][7][j])));
      if (den > 0.0f) c[cc] = __fdiv_rn(num, den);
    }
  }

  // --- final codes with the final c, packed into the staging buffer --------------------
  float ic[4];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) ic[cc] = recip_scale(c[cc]);
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const uint32_t info = sm.info[i];
    const int bits = row_bits(info);
    if (bits == PIVOT) continue;
    const float mb = sm.mb[i], q = sm.qm[i];
    uint32_t field = 0;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float t = __fmaf_rn(s[rr][cc], ic[cc], mb);
      t = fminf(fmaxf(t, mb - q), mb + q);
      const uint32_t u = __float_as_uint(t) & 0xFFu;
      field |= u << (bits * cc);
    }
    store_field(stage + row_off(info), bits, lane, field);
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) c_out[cc] = c[cc];
}

// ---------------------------------------------------------------------------------
// stq_decode_step: one CTA per (request, head).
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 2)
decode_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, const float* __restrict__ q,
              const float* __restrict__ k, const float* __restrict__ v,
              const float* __restrict__ gate, const float* __restrict__ beta,
              float* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ HeadSmem sm;
  const int item = blockIdx.x;
  const int bq = item / P.H, h = item - bq * P.H;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int slot = slots[bq];
  if (slot < 0 || slot >= P.n_slots) {
    if (tid == 0) atomicOr(P.err, ERR_SLOT_RANGE);
    return;
  }
  const HeadRef hr = head_ref(P, slot, h);
  const uint64_t vec = uint64_t(item) * D;

  // ---- load: per-row vectors, the head's packed codes and pivot rows ----------------
  load_row_meta(P, h, sm);
  if (tid < D) {
    sm.k[tid] = k[vec + tid];
    sm.q[tid] = q[vec + tid];
    sm.v[tid] = v[vec + tid];
    const float dec = (P.kind == 0) ? gate[item] : gate[vec + tid];
    sm.dec[tid] = dec;
    sm.rd[tid] = fmul(dec, hr.scales[tid]);
  }
  if (tid == 0) sm.beta = beta[item];
  copy16(stage, hr.codes, hr.code_bytes);
  copy16(stage + hr.piv_stage_off, hr.pivots, hr.piv_count * D * 2);
  float cin[4];
  {
    const float4 c4 = *reinterpret_cast<const float4*>(hr.scales + D + 4 * lane);
    cin[0] = c4.x; cin[1] = c4.y; cin[2] = c4.z; cin[3] = c4.w;
  }
  __syncthreads();

  // ---- restore S' = D (r c Q) and the column sums u_j = sum_i k_i S'_ij ---------------
  float s[RPW][4];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const uint32_t info = sm.info[i];
    const int bits = row_bits(info);
    if (bits == PIVOT) {
      const uint2 hv = *reinterpret_cast<const uint2*>(stage + hr.piv_stage_off + row_off(info) * (D * 2) + 8 * lane);
      const float dec = sm.dec[i];
      s[rr][0] = fmul(dec, __half2float(__ushort_as_half(uint16_t(hv.x & 0xFFFFu))));
      s[rr][1] = fmul(dec, __half2float(__ushort_as_half(uint16_t(hv.x >> 16))));
      s[rr][2] = fmul(dec, __half2float(__ushort_as_half(uint16_t(hv.y & 0xFFFFu))));
      s[rr][3] = fmul(dec, __half2float(__ushort_as_half(uint16_t(hv.y >> 16))));
    } else {
      const uint32_t f = lane_field(stage + row_off(info), bits, lane);
      const uint32_t mask = (1u << bits) - 1u;
      const float tb = TWO23 + float(1 << (bits - 1));
      const float rd = sm.rd[i];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const float Q = code_value((f >> (bits * cc)) & mask, tb);
        s[rr][cc] = fmul(fmul(Q, rd), cin[cc]);
      }
    }
  }
  {
    Vec<4> u = tree<0, RPW, 4>([&](int rr) {
      const float kk = sm.k[w * RPW + rr];
      Vec<4> leaf;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) leaf.x[cc] = fmul(kk, s[rr][cc]);
      return leaf;
    });
    *reinterpret_cast<float4*>(&sm.red[0][0][w][4 * lane]) = make_float4(u.x[0], u.x[1], u.x[2], u.x[3]);
  }
  __syncthreads();

  // ---- delta_j = beta (v_j - u_j); S = S' + k delta^T; readout partials ----------------
  float delta[4];
  {
    const float bt = sm.beta;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int j = 4 * lane + cc;
      float (*r0)[D] = sm.red[0][0];
      const float u = fadd(fadd(fadd(r0[0][j], r0[1][j]), fadd(r0[2][j], r0[3][j])),
                           fadd(fadd(r0[4][j], r0[5][j]), fadd(r0[6][j], r0[7][j])));
      delta[cc] = fmul(bt, __fsub_rn(sm.v[j], u));
    }
  }
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const float kk = sm.k[w * RPW + rr];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) s[rr][cc] = fadd(s[rr][cc], fmul(kk, delta[cc]));
  }
  {
    Vec<4> o = tree<0, RPW, 4>([&](int rr) {
      const float qq = sm.q[w * RPW + rr];
      Vec<4> leaf;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) leaf.x[cc] = fmul(qq, s[rr][cc]);
      return leaf;
    });
    *reinterpret_cast<float4*>(&sm.red[1][0][w][4 * lane]) = make_float4(o.x[0], o.x[1], o.x[2], o.x[3]);
  }
  // pivot rows: store float16(S) now (they take no part in the refit)
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const uint32_t info = sm.info[w * RPW + rr];
    if (row_bits(info) == PIVOT) {
      const uint32_t lo = uint32_t(__half_as_ushort(__float2half_rn(s[rr][0]))) |
                          (uint32_t(__half_as_ushort(__float2half_rn(s[rr][1]))) << 16);
      const uint32_t hi = uint32_t(__half_as_ushort(__float2half_rn(s[rr][2]))) |
                          (uint32_t(__half_as_ushort(__float2half_rn(s[rr][3]))) << 16);
      *reinterpret_cast<uint2*>(hr.pivots + row_off(info) * D + 4 * lane) = make_uint2(lo, hi);
    }
  }

  // ---- refit + requantise (all-pivot heads keep r = c = 0) ---------------------------
  float c[4];
  if (hr.piv_count == D) {
    __syncthreads();
    if (w == 0) {
      float o[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int j = 4 * lane + cc;
        float (*r1)[D] = sm.red[1][0];
        o[cc] = fadd(fadd(fadd(r1[0][j], r1[1][j]), fadd(r1[2][j], r1[3][j])),
                     fadd(fadd(r1[4][j], r1[5][j]), fadd(r1[6][j], r1[7][j])));
      }
      *reinterpret_cast<float4*>(out + vec + 4 * lane) = make_float4(o[0], o[1], o[2], o[3]);
    }
    if (tid < D) hr.scales[tid] = 0.0f;
    c[0] = c[1] = c[2] = c[3] = 0.0f;
  } else {
    refit_pack(P, h, sm, stage, s, hr.scales, c, out + vec);
  }
  __syncthreads();
  copy16_out(hr.codes, stage, hr.code_bytes);
  if (w == 0) *reinterpret_cast<float4*>(hr.scales + D + 4 * lane) = make_float4(c[0], c[1], c[2], c[3]);
}

// ---------------------------------------------------------------------------------
// stq_quantize_init: float32 states -> packed pool.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 2)
quantize_kernel(PoolDev P, const int32_t* __restrict__ slots, int B, const float* __restrict__ S) {
  extern __shared__ __align__(16) uint8_t stage[];
  __shared__ HeadSmem sm;
  const int item = blockIdx.x;
  const int bq = item / P.H, h = item - bq * P.H;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int slot = slots[bq];
  if (slot < 0 || slot >= P.n_slots) {
    if (tid == 0) atomicOr(P.err, ERR_SLOT_RANGE);
    return;
  }
  const HeadRef hr = head_ref(P, slot, h);
  load_row_meta(P, h, sm);
  __syncthreads();
  float s[RPW][4];
  const float* src = S + uint64_t(item) * D * D;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const float4 x = *reinterpret_cast<const float4*>(src + i * D + 4 * lane);
    s[rr][0] = x.x; s[rr][1] = x.y; s[rr][2] = x.z; s[rr][3] = x.w;
    const uint32_t info = sm.info[i];
    if (row_bits(info) == PIVOT) {
      const uint32_t lo = uint32_t(__half_as_ushort(__float2half_rn(x.x))) |
                          (uint32_t(__half_as_ushort(__float2half_rn(x.y))) << 16);
      const uint32_t hi = uint32_t(__half_as_ushort(__float2half_rn(x.z))) |
                          (uint32_t(__half_as_ushort(__float2half_rn(x.w))) << 16);
      *reinterpret_cast<uint2*>(hr.pivots + row_off(info) * D + 4 * lane) = make_uint2(lo, hi);
    }
  }
  float c[4];
  if (hr.piv_count == D) {
    if (tid < D) hr.scales[tid] = 0.0f;
    c[0] = c[1] = c[2] = c[3] = 0.0f;
  } else {
    refit_pack(P, h, sm, stage, s, hr.scales, c, nullptr);
  }
  __syncthreads();
  copy16_out(hr.codes, stage, hr.code_bytes);
  if (w == 0) *reinterpret_cast<float4*>(hr.scales + D + 4 * lane) = make_float4(c[0], c[1], c[2], c[3]);
}

// ---------------------------------------------------------------------------------
// stq_dequantize: packed pool -> float32 states, S_ij = (Q_ij r_i) c_j.
// ---------------------------------------------------------------------------------
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
  const float cin[4] = {c4.x, c4.y, c4.z, c4.w};
  __syncthreads();
  float* dst = S_out + uint64_t(item) * D * D;
#pragma unroll 4
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const uint32_t info = info_s[i];
    const int bits = row_bits(info);
    float x[4];
    if (bits == PIVOT) {
      const uint2 hv = *reinterpret_cast<const uint2*>(stage + hr.piv_stage_off + row_off(info) * (D * 2) + 8 * lane);
      x[0] = __half2float(__ushort_as_half(uint16_t(hv.x & 0xFFFFu)));
      x[1] = __half2float(__ushort_as_half(uint16_t(hv.x >> 16)));
      x[2] = __half2float(__ushort_as_half(uint16_t(hv.y & 0xFFFFu)));
      x[3] = __half2float(__ushort_as_half(uint16_t(hv.y >> 16)));
    } else {
      const uint32_t f = lane_field(stage + row_off(info), bits, lane);
      const uint32_t mask = (1u << bits) - 1u;
      const float tb = TWO23 + float(1 << (bits - 1));
      const float r = r_s[i];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) x[cc] = fmul(fmul(code_value((f >> (bits * cc)) & mask, tb), r), cin[cc]);
    }
    *reinterpret_cast<float4*>(dst + i * D + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
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
  __shared__ float ks[D], qs[D], vs[D], ds[D];
  __shared__ __align__(16) float red[2][NW][D];
  const int item = blockIdx.x;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
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
  float s[RPW][4];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const float4 x = *reinterpret_cast<const float4*>(base + i * D + 4 * lane);
    const float dd = ds[i];
    s[rr][0] = fmul(dd, x.x); s[rr][1] = fmul(dd, x.y); s[rr][2] = fmul(dd, x.z); s[rr][3] = fmul(dd, x.w);
  }
  Vec<4> u = tree<0, RPW, 4>([&](int rr) {
    const float kk = ks[w * RPW + rr];
    Vec<4> leaf;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) leaf.x[cc] = fmul(kk, s[rr][cc]);
    return leaf;
  });
  *reinterpret_cast<float4*>(&red[0][w][4 * lane]) = make_float4(u.x[0], u.x[1], u.x[2], u.x[3]);
  __syncthreads();
  float delta[4];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int j = 4 * lane + cc;
    const float uu = fadd(fadd(fadd(red[0][0][j], red[0][1][j]), fadd(red[0][2][j], red[0][3][j])),
                          fadd(fadd(red[0][4][j], red[0][5][j]), fadd(red[0][6][j], red[0][7][j])));
    delta[cc] = fmul(bt, __fsub_rn(vs[j], uu));
  }
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int i = w * RPW + rr;
    const float kk = ks[i];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) s[rr][cc] = fadd(s[rr][cc], fmul(kk, delta[cc]));
    *reinterpret_cast<float4*>(base + i * D + 4 * lane) = make_float4(s[rr][0], s[rr][1], s[rr][2], s[rr][3]);
  }
  Vec<4> o = tree<0, RPW, 4>([&](int rr) {
    const float qq = qs[w * RPW + rr];
    Vec<4> leaf;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) leaf.x[cc] = fmul(qq, s[rr][cc]);
    return leaf;
  });
  *reinterpret_cast<float4*>(&red[1][w][4 * lane]) = make_float4(o.x[0], o.x[1], o.x[2], o.x[3]);
  __syncthreads();
  if (w == 0) {
    float oo[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const int j = 4 * lane + cc;
      oo[cc] = fadd(fadd(fadd(red[1][0][j], red[1][1][j]), fadd(red[1][2][j], red[1][3][j])),
                    fadd(fadd(red[1][4][j], red[1][5][j]), fadd(red[1][6][j], red[1][7][j])));
    }
    *reinterpret_cast<float4*>(out + vec + 4 * lane) = make_float4(oo[0], oo[1], oo[2], oo[3]);
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

int g_decode_dyn[64], g_quant_dyn[64], g_dequant_dyn[64];

}  // namespace

cudaError_t launch_decode(const PoolDev& P, const int32_t* slots, int B, const float* q,
                          const float* k, const float* v, const float* gate,
                          const float* beta, float* out, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const int dyn = stage_bytes(P);
  cudaError_t e = prepare(decode_kernel, dyn, int(sizeof(HeadSmem)), g_decode_dyn);
  if (e != cudaSuccess) return e;
  decode_kernel<<<B * P.H, NT, dyn, s>>>(P, slots, B, q, k, v, gate, beta, out);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const PoolDev& P, const int32_t* slots, int B, const float* S,
                            cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const int dyn = stage_bytes(P);
  cudaError_t e = prepare(quantize_kernel, dyn, int(sizeof(HeadSmem)), g_quant_dyn);
  if (e != cudaSuccess) return e;
  quantize_kernel<<<B * P.H, NT, dyn, s>>>(P, slots, B, S);
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
