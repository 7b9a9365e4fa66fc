// Offline calibration of a pool's widths: the per-row reconstruction error kernel
// (device) and the lifetime weights, unit distortions and budgeted width allocation
// (host). The method: lifetime weight L_u = sum_{j<J} exp(2 j l_u) (bloombook section
// 3), widths minimising the lifetime-weighted distortion under a mean-bit budget with
// a few FP16 pivot units (bloombook section 4; singularity-lens calibration paragraph).
#include <cmath>
#include <cstdio>
#include <limits>
#include <vector>

#include <cuda_fp16.h>

#include "stq.h"
#include "stq_internal.h"

namespace {

constexpr int kD = 128;

// One warp per row: lane l squares the differences of columns 4l..4l+3, adds them as
// (c0 + c1) + (c2 + c3), and the lanes meet in butterfly steps xor 1, 2, 4, 8, 16 --
// a balanced binary tree over the 128 columns.
__global__ void __launch_bounds__(256)
row_sq_error_kernel(const float4* __restrict__ S, const float4* __restrict__ S_hat, long long n_rows,
                    float* __restrict__ err, int accumulate) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const float4 a = S[row * 32 + lane];
  const float4 b = S_hat[row * 32 + lane];
  const float d0 = __fsub_rn(a.x, b.x), d1 = __fsub_rn(a.y, b.y);
  const float d2 = __fsub_rn(a.z, b.z), d3 = __fsub_rn(a.w, b.w);
  float e = __fadd_rn(__fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1)),
                      __fadd_rn(__fmul_rn(d2, d2), __fmul_rn(d3, d3)));
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) e = __fadd_rn(e, __shfl_xor_sync(0xffffffffu, e, m));
  if (lane == 0) err[row] = accumulate ? __fadd_rn(err[row], e) : e;
}

// In-head distortion of a row at candidate widths: one warp per row of one (state, head)
// of a quantised pool. The row keeps the refit's row scale r_i (computed here from S for
// every row, pivot rows included) and the head's stored column scales c_j; only the
// reach of its codes changes with the width: Q = clamp(rint((S r^-1) c^-1), +-qmax_b)
// on the exact product, S_hat = (Q r) c, and the error is the tree sum of the squared
// differences (the row_sq_error_kernel's tree).
struct CandWidths {
  int n;
  float qmax[4];
};

template <bool H16>
__global__ void __launch_bounds__(256)
row_error_at_widths_kernel(stq::PoolDev P, const int32_t* __restrict__ slots, int B,
                           const float4* __restrict__ S, CandWidths cw, float* __restrict__ err) {
  constexpr float kMagic = 12582912.0f;            // 1.5 * 2^23
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long n_rows = (long long)B * P.H * kD;
  if (row >= n_rows) return;
  const long long hs = row / kD;                   // (state, head)
  const int i = int(row - hs * kD);
  const int n = int(hs / P.H), h = int(hs - (long long)n * P.H);
  const int slot = slots[n];
  if (slot < 0 || slot >= P.n_slots) {
    if (lane == 0 && i == 0) atomicOr(P.err, stq::ERR_SLOT_RANGE);
    return;
  }
  const size_t cbase = (size_t(slot) * P.H + h) * 2 * kD + kD + 4 * lane;
  float c[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if constexpr (H16) c[e] = __half2float(static_cast<const __half*>(P.scales)[cbase + e]);
    else c[e] = static_cast<const float*>(P.scales)[cbase + e];
  }
  const float4 x = S[row * 32 + lane];
  const float sv[4] = {x.x, x.y, x.z, x.w};
  float a = __fadd_rn(__fadd_rn(fabsf(sv[0]), fabsf(sv[1])), __fadd_rn(fabsf(sv[2]), fabsf(sv[3])));
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, m));
  float r = __fmul_rn(__fmul_rn(a, 0.0078125f), P.g[h * kD + i]);
  if constexpr (H16) r = __half2float(__float2half_rn(r));   // a compact pool stores r as binary16
  const float tiny = 1.17549435e-38f;              // scales below 2^-126 count as zero
  const float ir = r >= tiny ? __frcp_rn(r) : 0.0f;
  float y[4], ic[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    y[e] = __fmul_rn(sv[e], ir);
    ic[e] = c[e] >= tiny ? __frcp_rn(c[e]) : 0.0f;
  }
  for (int ci = 0; ci < cw.n; ++ci) {
    const float lo = kMagic - cw.qmax[ci], hi = kMagic + cw.qmax[ci];
    float d2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float t = fminf(fmaxf(__fmaf_rn(y[e], ic[e], kMagic), lo), hi);
      const float q = __fadd_rn(t, -kMagic);
      const float d = __fsub_rn(sv[e], __fmul_rn(__fmul_rn(q, r), c[e]));
      d2[e] = __fmul_rn(d, d);
    }
    float ev = __fadd_rn(__fadd_rn(d2[0], d2[1]), __fadd_rn(d2[2], d2[3]));
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) ev = __fadd_rn(ev, __shfl_xor_sync(0xffffffffu, ev, m));
    if (lane == 0) err[row * cw.n + ci] = ev;
  }
}

stq_status fail(stq_status st, const char* msg) {
  stq::set_last_error(msg);
  return st;
}

stq_status ok() {
  stq::clear_last_error();
  return STQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" stq_status stq_row_sq_error(const float* d_S, const float* d_S_hat, int n_states,
                                       float* d_err, int accumulate, void* stream) {
  if (n_states < 0) return fail(STQ_ERR_INVALID_ARG, "n_states must be >= 0");
  if (n_states == 0) return ok();
  if (!d_S || !d_S_hat || !d_err) return fail(STQ_ERR_INVALID_ARG, "a device pointer is NULL");
  if (!aligned16(d_S) || !aligned16(d_S_hat) || !aligned16(d_err))
    return fail(STQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  const long long n_rows = (long long)n_states * kD;
  const long long blocks = (n_rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return fail(STQ_ERR_INVALID_ARG, "n_states too large");
  row_sq_error_kernel<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4*>(d_S), reinterpret_cast<const float4*>(d_S_hat), n_rows, d_err,
      accumulate);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char buf[256];
    snprintf(buf, sizeof(buf), "stq_row_sq_error launch: %s", cudaGetErrorString(e));
    return fail(STQ_ERR_CUDA, buf);
  }
  return ok();
}

extern "C" stq_status stq_row_error_at_widths(stq_pool* pool, const int32_t* d_slots, int B,
                                              const float* d_S, const int* h_cand_bits, int n_cand,
                                              float* d_err, void* stream) {
  const int st = stq::check_batch(pool, d_slots, B);
  if (st != STQ_OK) return static_cast<stq_status>(st);
  if (h_cand_bits == nullptr || n_cand < 1 || n_cand > 4)
    return fail(STQ_ERR_INVALID_ARG, "need 1 to 4 candidate widths");
  CandWidths cw;
  cw.n = n_cand;
  for (int k = 0; k < n_cand; ++k) {
    const int b = h_cand_bits[k];
    if (b != 2 && b != 4 && b != 6 && b != 8) return fail(STQ_ERR_INVALID_ARG, "candidate width not in {2,4,6,8}");
    cw.qmax[k] = float((1 << (b - 1)) - 1);
  }
  for (int k = n_cand; k < 4; ++k) cw.qmax[k] = 0.0f;
  if (B == 0) return ok();
  if (!d_S || !d_err) return fail(STQ_ERR_INVALID_ARG, "a device pointer is NULL");
  if (!aligned16(d_S) || !aligned16(d_err)) return fail(STQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  const stq::PoolDev* P = stq::pool_dev(pool);
  const long long n_rows = (long long)B * P->H * kD;
  const long long blocks = (n_rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return fail(STQ_ERR_INVALID_ARG, "B too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float4* S4 = reinterpret_cast<const float4*>(d_S);
  if (P->scale16) row_error_at_widths_kernel<true><<<unsigned(blocks), 256, 0, s>>>(*P, d_slots, B, S4, cw, d_err);
  else row_error_at_widths_kernel<false><<<unsigned(blocks), 256, 0, s>>>(*P, d_slots, B, S4, cw, d_err);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char buf[256];
    snprintf(buf, sizeof(buf), "stq_row_error_at_widths launch: %s", cudaGetErrorString(e));
    return fail(STQ_ERR_CUDA, buf);
  }
  return ok();
}

extern "C" stq_status stq_lifetime_weights(const double* ell, int n, int horizon, double* out) {
  if (n < 0 || horizon < 1) return fail(STQ_ERR_INVALID_ARG, "need n >= 0 and horizon >= 1");
  if (n > 0 && (!ell || !out)) return fail(STQ_ERR_INVALID_ARG, "a host pointer is NULL");
  for (int u = 0; u < n; ++u) {
    if (!(ell[u] <= 0.0)) return fail(STQ_ERR_INVALID_ARG, "a mean log-retention is > 0 or NaN");
    double acc = 0.0;
    for (int j = 0; j < horizon; ++j) acc += std::exp(2.0 * double(j) * ell[u]);
    out[u] = acc;
  }
  return ok();
}

extern "C" stq_status stq_unit_distortion(int kind, int N, int H, const float* h_row_err,
                                          const float* h_omega, double* out) {
  if (kind != STQ_GDN && kind != STQ_KDA) return fail(STQ_ERR_INVALID_ARG, "bad kind");
  if (N <= 0 || H <= 0) return fail(STQ_ERR_INVALID_ARG, "need N > 0 and H > 0");
  if (!h_row_err || !out || (kind == STQ_GDN && !h_omega))
    return fail(STQ_ERR_INVALID_ARG, "a host pointer is NULL");
  if (kind == STQ_GDN) {
    for (int h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int n = 0; n < N; ++n)
        for (int i = 0; i < kD; ++i)
          acc += double(h_omega[size_t(h) * kD + i]) * double(h_row_err[(size_t(n) * H + h) * kD + i]);
      out[h] = acc / double(N * kD * kD);
    }
  } else {
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < kD; ++i) {
        double acc = 0.0;
        for (int n = 0; n < N; ++n) acc += double(h_row_err[(size_t(n) * H + h) * kD + i]);
        out[size_t(h) * kD + i] = acc / double(N * kD);
      }
  }
  return ok();
}

extern "C" stq_status stq_allocate_bits(int n, int n_cand, const int* cand_bits, const double* lifetime,
                                        const double* dist, double budget, int n_pivots,
                                        uint8_t* out_bits) {
  if (n < 0 || n_cand < 1 || n_cand > 4 || n_pivots < 0 || n_pivots > n)
    return fail(STQ_ERR_INVALID_ARG, "need n >= 0, 1 <= n_cand <= 4, 0 <= n_pivots <= n");
  if (!cand_bits || (n > 0 && (!lifetime || !dist || !out_bits)))
    return fail(STQ_ERR_INVALID_ARG, "a host pointer is NULL");
  for (int c = 0; c < n_cand; ++c) {
    const int b = cand_bits[c];
    if (b != 2 && b != 4 && b != 6 && b != 8) return fail(STQ_ERR_INVALID_ARG, "candidate width not in {2,4,6,8}");
    if (c > 0 && b <= cand_bits[c - 1]) return fail(STQ_ERR_INVALID_ARG, "candidate widths must ascend");
  }
  // costs and pivots: the n_pivots largest risks lifetime * dist(widest)
  std::vector<double> cost(size_t(n) * n_cand);
  for (int u = 0; u < n; ++u)
    for (int c = 0; c < n_cand; ++c) cost[size_t(u) * n_cand + c] = lifetime[u] * dist[size_t(u) * n_cand + c];
  std::vector<char> pivot(n, 0);
  for (int p = 0; p < n_pivots; ++p) {
    int pick = -1;
    for (int u = 0; u < n; ++u) {
      if (pivot[u]) continue;
      if (pick < 0 || cost[size_t(u) * n_cand + n_cand - 1] > cost[size_t(pick) * n_cand + n_cand - 1]) pick = u;
    }
    pivot[pick] = 1;
  }
  std::vector<int> rest;
  for (int u = 0; u < n; ++u)
    if (!pivot[u]) rest.push_back(u);
  const int m = int(rest.size());
  const int K = int(std::floor(budget * double(m) / 2.0));
  const int k0 = cand_bits[0] / 2;
  if (!(budget >= 0.0) || (long long)k0 * m > K)
    return fail(STQ_ERR_INVALID_ARG, "budget below the narrowest candidate width");
  // dynamic program over the total width in steps of 2 bits
  const double inf = std::numeric_limits<double>::infinity();
  std::vector<double> best(size_t(K) + 1, inf), next(size_t(K) + 1);
  std::vector<signed char> choice(size_t(m) * (size_t(K) + 1));
  best[0] = 0.0;
  for (int t = 0; t < m; ++t) {
    const int u = rest[t];
    signed char* ch = &choice[size_t(t) * (size_t(K) + 1)];
    for (int s = 0; s <= K; ++s) {
      next[s] = inf;
      ch[s] = -1;
    }
    for (int c = 0; c < n_cand; ++c) {
      const int k = cand_bits[c] / 2;
      const double cu = cost[size_t(u) * n_cand + c];
      for (int s = k; s <= K; ++s) {
        const double v = best[s - k] + cu;
        if (v < next[s]) {
          next[s] = v;
          ch[s] = static_cast<signed char>(c);
        }
      }
    }
    best.swap(next);
  }
  int s = 0;
  for (int t = 1; t <= K; ++t)
    if (best[t] < best[s]) s = t;
  for (int u = 0; u < n; ++u) out_bits[u] = STQ_PIVOT_BITS;
  for (int t = m - 1; t >= 0; --t) {
    const int c = choice[size_t(t) * (size_t(K) + 1) + s];
    out_bits[rest[t]] = static_cast<uint8_t>(cand_bits[c]);
    s -= cand_bits[c] / 2;
  }
  return ok();
}
