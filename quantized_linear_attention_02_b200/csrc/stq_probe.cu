// Issue-rate probe: a kernel of independent register-only chains of one instruction kind,
// so that a caller timing it with CUDA events measures the rate at which the SMs retire
// that kind (lane operations per second). The decode step is bound by instruction issue
// on the CUDA cores, and this is the measured rate its roofline is set against.
#include <cstdio>

#include "stq.h"
#include "stq_internal.h"

namespace {

constexpr int kProbeThreads = 512;
constexpr int kChains = 8;   // independent chains per thread (enough to cover the latency)

// mode 0: packed fma.rn.f32x2 (2 lane operations each); 1: scalar fma.rn.f32;
// 2: lop3.b32 (integer logic on the ALU pipe). Every chain's result reaches `out`.
__global__ void __launch_bounds__(kProbeThreads) issue_rate_kernel(float* __restrict__ out, int mode, int iters) {
  const float t = float(threadIdx.x) * 1.0e-6f;
  float r = 0.0f;
  if (mode == 0) {
    float2 a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = make_float2(t + float(i), t - float(i));
    const float2 m = make_float2(0.999f + t, 0.998f - t), c = make_float2(1.0e-3f, t);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) a[i] = __ffma2_rn(a[i], m, c);
    }
#pragma unroll
    for (int i = 0; i < kChains; ++i) r += a[i].x + a[i].y;
  } else if (mode == 1) {
    float a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = t + float(i);
    const float m = 0.999f + t, c = 1.0e-3f;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) a[i] = __fmaf_rn(a[i], m, c);
    }
#pragma unroll
    for (int i = 0; i < kChains; ++i) r += a[i];
  } else {
    uint32_t a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) a[i] = threadIdx.x * 2654435761u + uint32_t(i);
    const uint32_t y = 0x9E3779B9u ^ threadIdx.x, z = 0x7F4A7C15u + blockIdx.x;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < kChains; ++i) asm volatile("lop3.b32 %0, %0, %1, %2, 0x96;" : "+r"(a[i]) : "r"(y), "r"(z));
    }
    uint32_t x = 0;
#pragma unroll
    for (int i = 0; i < kChains; ++i) x ^= a[i];
    r = float(x & 0xFFFFu);
  }
  out[size_t(blockIdx.x) * kProbeThreads + threadIdx.x] = r;
}

stq_status probe_fail(stq_status st, const char* msg) {
  stq::set_last_error(msg);
  return st;
}

}  // namespace

extern "C" stq_status stq_issue_rate_probe(int mode, int blocks, int iters, float* d_out, void* stream) {
  if (mode < 0 || mode > 2) return probe_fail(STQ_ERR_INVALID_ARG, "mode must be 0, 1 or 2");
  if (blocks < 1 || blocks > 65535) return probe_fail(STQ_ERR_INVALID_ARG, "blocks must be in [1, 65535]");
  if (iters < 1) return probe_fail(STQ_ERR_INVALID_ARG, "iters must be >= 1");
  if (d_out == nullptr) return probe_fail(STQ_ERR_INVALID_ARG, "d_out is NULL");
  issue_rate_kernel<<<unsigned(blocks), kProbeThreads, 0, static_cast<cudaStream_t>(stream)>>>(d_out, mode, iters);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char buf[160];
    snprintf(buf, sizeof(buf), "stq_issue_rate_probe launch: %s", cudaGetErrorString(e));
    return probe_fail(STQ_ERR_CUDA, buf);
  }
  stq::clear_last_error();
  return STQ_OK;
}
