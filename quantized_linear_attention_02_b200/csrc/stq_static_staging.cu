// stq_decode_step_host_static: the host-buffer decode step with its device staging in
// a fixed array declared here instead of a caller-provided buffer, for callers that
// cannot allocate device memory on their decode path.
#include <cstdio>
#include <mutex>

#include "stq.h"
#include "stq_internal.h"

namespace {

// The staging array. In host code this name is only a host-side stand-in for the
// device symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_static_staging[STQ_STATIC_STAGING_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_staging_addr[kMaxDevices];   // device address of g_static_staging, per device

// Device address of the staging array on the current device (looked up once per device).
cudaError_t staging_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_staging_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_staging);
    if (e != cudaSuccess) return e;
    g_staging_addr[dev] = p;
  }
  *out = g_staging_addr[dev];
  return cudaSuccess;
}

stq_status fail(stq_status st, const char* msg) {
  stq::set_last_error(msg);
  return st;
}

}  // namespace

extern "C" stq_status stq_decode_step_host_static(stq_pool* pool, const int32_t* d_slots, int B,
                                                  const float* h_q, const float* h_k,
                                                  const float* h_v, const float* h_gate,
                                                  const float* h_beta, float* h_out,
                                                  void* stream) {
  const int st = stq::check_batch(pool, d_slots, B);
  if (st != STQ_OK) return static_cast<stq_status>(st);
  if (B == 0) {
    stq::clear_last_error();
    return STQ_OK;
  }
  if (!h_q || !h_k || !h_v || !h_gate || !h_beta || !h_out)
    return fail(STQ_ERR_INVALID_ARG, "a host pointer is NULL");
  const stq::PoolDev* P = stq::pool_dev(pool);
  const stq::StagingLayout L = stq::staging_layout(*P, B);
  if (L.total > STQ_STATIC_STAGING_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "B=%d x H=%d needs %zu bytes of staging, more than the static %u; "
             "use stq_decode_step_host with a caller buffer", B, P->H, L.total,
             unsigned(STQ_STATIC_STAGING_BYTES));
    return fail(STQ_ERR_INVALID_ARG, msg);
  }
  void* base_v = nullptr;
  cudaError_t e = staging_address(&base_v);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "device address of the static staging: %s", cudaGetErrorString(e));
    return fail(STQ_ERR_CUDA, msg);
  }
  uint8_t* base = static_cast<uint8_t*>(base_v);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* dq = reinterpret_cast<float*>(base + L.q);
  float* dk = reinterpret_cast<float*>(base + L.k);
  float* dv = reinterpret_cast<float*>(base + L.v);
  float* dg = reinterpret_cast<float*>(base + L.gate);
  float* db = reinterpret_cast<float*>(base + L.beta);
  float* dout = reinterpret_cast<float*>(base + L.out);
  struct Copy { void* dst; const void* src; size_t n; };
  const Copy in[] = {{dq, h_q, L.n_vec * 4}, {dk, h_k, L.n_vec * 4}, {dv, h_v, L.n_vec * 4},
                     {dg, h_gate, L.n_gate * 4}, {db, h_beta, L.n_beta * 4}};
  for (const Copy& c : in) {
    e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof(msg), "host-to-device copy of step inputs: %s", cudaGetErrorString(e));
      return fail(STQ_ERR_CUDA, msg);
    }
  }
  e = stq::launch_decode(*P, d_slots, B, dq, dk, dv, dg, db, dout, s);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "stq_decode_step launch: %s", cudaGetErrorString(e));
    return fail(STQ_ERR_CUDA, msg);
  }
  e = cudaMemcpyAsync(h_out, dout, L.n_vec * 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "device-to-host copy of the readout: %s", cudaGetErrorString(e));
    return fail(STQ_ERR_CUDA, msg);
  }
  stq::clear_last_error();
  return STQ_OK;
}
