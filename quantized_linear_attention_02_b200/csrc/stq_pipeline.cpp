// The host-buffer decode step pipelined two deep inside the library: step i's inputs go
// up on an upload stream while step i-1 decodes, and step i's readout comes down on a
// download stream while step i+1 decodes. The decode steps themselves stay in order on
// the caller's stream (each reads the state the previous one wrote). Two halves of a
// caller-allocated staging buffer alternate between steps; events order every reuse.
#include <cstdio>
#include <new>

#include "stq.h"
#include "stq_internal.h"

namespace {

stq_status fail(stq_status st, const char* msg) {
  stq::set_last_error(msg);
  return st;
}

stq_status cuda_fail(cudaError_t e, const char* what) {
  char msg[256];
  snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
  return fail(STQ_ERR_CUDA, msg);
}

struct Half {
  float *q, *k, *v, *gate, *beta, *out;
  cudaEvent_t inputs_read;   // the decode that read this half's inputs has finished
  cudaEvent_t uploaded;      // this half's inputs are on the device
  cudaEvent_t decoded;       // the decode that wrote this half's readout has finished
  cudaEvent_t downloaded;    // this half's readout is on the host
};

}  // namespace

struct stq_pipeline {
  stq_pool* pool = nullptr;
  int B = 0;
  size_t n_vec = 0, n_gate = 0, n_bh = 0;
  int device = 0;
  cudaStream_t up = nullptr, down = nullptr;
  Half half[2] = {};
  long long steps = 0;       // steps enqueued so far
  bool used[2] = {false, false};
};

namespace {

void destroy_events(stq_pipeline* p) {
  for (Half& h : p->half) {
    for (cudaEvent_t* e : {&h.inputs_read, &h.uploaded, &h.decoded, &h.downloaded})
      if (*e) cudaEventDestroy(*e), *e = nullptr;
  }
}

}  // namespace

extern "C" {

size_t stq_pipeline_staging_bytes(const stq_pool* pool, int B) {
  const stq::PoolDev* P = stq::pool_dev(pool);
  if (P == nullptr || B < 0) return 0;
  return 2 * stq::staging_layout(*P, B).total;
}

stq_status stq_pipeline_create(stq_pool* pool, int B, void* d_staging, size_t staging_bytes,
                               stq_pipeline** out) {
  if (out == nullptr) return fail(STQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (B <= 0) return fail(STQ_ERR_INVALID_ARG, "B must be > 0");
  const int32_t one_slot = 0;   // check_batch only tests d_slots for NULL here
  const int st = stq::check_batch(pool, &one_slot, B);
  if (st != STQ_OK) return static_cast<stq_status>(st);
  const stq::PoolDev* P = stq::pool_dev(pool);
  if (d_staging == nullptr) return fail(STQ_ERR_INVALID_ARG, "d_staging is NULL");
  if ((reinterpret_cast<uintptr_t>(d_staging) & 15u) != 0)
    return fail(STQ_ERR_ALIGNMENT, "d_staging must be 16-byte aligned");
  const stq::StagingLayout L = stq::staging_layout(*P, B);
  const size_t hb = L.total;
  const size_t offs[6] = {L.q, L.k, L.v, L.gate, L.beta, L.out};
  if (staging_bytes < 2 * hb) {
    char msg[160];
    snprintf(msg, sizeof(msg), "staging_bytes %zu < %zu (stq_pipeline_staging_bytes)", staging_bytes, 2 * hb);
    return fail(STQ_ERR_INVALID_ARG, msg);
  }
  stq_pipeline* p = new (std::nothrow) stq_pipeline();
  if (p == nullptr) return fail(STQ_ERR_INVALID_ARG, "out of host memory");
  p->pool = pool;
  p->B = B;
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->up, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->down, cudaStreamNonBlocking);
  uint8_t* base = static_cast<uint8_t*>(d_staging);
  for (int j = 0; j < 2 && e == cudaSuccess; ++j) {
    Half& h = p->half[j];
    uint8_t* b = base + j * hb;
    h.q = reinterpret_cast<float*>(b + offs[0]);
    h.k = reinterpret_cast<float*>(b + offs[1]);
    h.v = reinterpret_cast<float*>(b + offs[2]);
    h.gate = reinterpret_cast<float*>(b + offs[3]);
    h.beta = reinterpret_cast<float*>(b + offs[4]);
    h.out = reinterpret_cast<float*>(b + offs[5]);
    for (cudaEvent_t* ev : {&h.inputs_read, &h.uploaded, &h.decoded, &h.downloaded})
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    destroy_events(p);
    if (p->up) cudaStreamDestroy(p->up);
    if (p->down) cudaStreamDestroy(p->down);
    delete p;
    return cuda_fail(e, "pipeline streams and events");
  }
  p->n_bh = L.n_beta;
  p->n_vec = L.n_vec;
  p->n_gate = L.n_gate;
  *out = p;
  stq::clear_last_error();
  return STQ_OK;
}

stq_status stq_pipeline_step(stq_pipeline* p, const int32_t* d_slots, const float* h_q,
                             const float* h_k, const float* h_v, const float* h_gate,
                             const float* h_beta, float* h_out, void* stream) {
  if (p == nullptr) return fail(STQ_ERR_INVALID_ARG, "pipeline is NULL");
  if (d_slots == nullptr) return fail(STQ_ERR_INVALID_ARG, "d_slots is NULL");
  if (!h_q || !h_k || !h_v || !h_gate || !h_beta || !h_out)
    return fail(STQ_ERR_INVALID_ARG, "a host pointer is NULL");
  const stq::PoolDev* P = stq::pool_dev(p->pool);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int j = int(p->steps & 1);
  Half& h = p->half[j];
  cudaError_t e = cudaSuccess;
  // upload: after the decode two steps back has read this half's inputs
  if (p->used[j]) e = cudaStreamWaitEvent(p->up, h.inputs_read, 0);
  struct Copy { void* dst; const void* src; size_t n; };
  const Copy in[] = {{h.q, h_q, p->n_vec * 4}, {h.k, h_k, p->n_vec * 4}, {h.v, h_v, p->n_vec * 4},
                     {h.gate, h_gate, p->n_gate * 4}, {h.beta, h_beta, p->n_bh * 4}};
  for (const Copy& c : in)
    if (e == cudaSuccess) e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, p->up);
  if (e == cudaSuccess) e = cudaEventRecord(h.uploaded, p->up);
  if (e != cudaSuccess) return cuda_fail(e, "pipeline upload");
  // decode on the caller's stream, after the inputs arrived and the readout of two steps
  // back left this half
  e = cudaStreamWaitEvent(s, h.uploaded, 0);
  if (e == cudaSuccess && p->used[j]) e = cudaStreamWaitEvent(s, h.downloaded, 0);
  if (e != cudaSuccess) return cuda_fail(e, "pipeline ordering");
  e = stq::launch_decode(*P, d_slots, p->B, h.q, h.k, h.v, h.gate, h.beta, h.out, s);
  if (e != cudaSuccess) return cuda_fail(e, "stq_decode_step launch");
  e = cudaEventRecord(h.inputs_read, s);
  if (e == cudaSuccess) e = cudaEventRecord(h.decoded, s);
  // download the readout
  if (e == cudaSuccess) e = cudaStreamWaitEvent(p->down, h.decoded, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(h_out, h.out, p->n_vec * 4, cudaMemcpyDeviceToHost, p->down);
  if (e == cudaSuccess) e = cudaEventRecord(h.downloaded, p->down);
  if (e != cudaSuccess) return cuda_fail(e, "pipeline download");
  p->used[j] = true;
  ++p->steps;
  // the previous step's readout: wait for it on the host
  if (p->steps >= 2) {
    e = cudaEventSynchronize(p->half[j ^ 1].downloaded);
    if (e != cudaSuccess) return cuda_fail(e, "waiting for the previous readout");
  }
  stq::clear_last_error();
  return STQ_OK;
}

stq_status stq_pipeline_finish(stq_pipeline* p, void* stream) {
  if (p == nullptr) return fail(STQ_ERR_INVALID_ARG, "pipeline is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  for (int j = 0; j < 2 && e == cudaSuccess; ++j) {
    if (!p->used[j]) continue;
    e = cudaStreamWaitEvent(s, p->half[j].downloaded, 0);
    if (e == cudaSuccess) e = cudaEventSynchronize(p->half[j].downloaded);
  }
  if (e != cudaSuccess) return cuda_fail(e, "pipeline finish");
  stq::clear_last_error();
  return STQ_OK;
}

void stq_pipeline_destroy(stq_pipeline* p) {
  if (p == nullptr) return;
  int cur = 0;
  const bool other = cudaGetDevice(&cur) == cudaSuccess && cur != p->device;
  if (other) cudaSetDevice(p->device);
  if (p->up) cudaStreamSynchronize(p->up);
  if (p->down) cudaStreamSynchronize(p->down);
  destroy_events(p);
  if (p->up) cudaStreamDestroy(p->up);
  if (p->down) cudaStreamDestroy(p->down);
  if (other) cudaSetDevice(cur);
  delete p;
}

}  // extern "C"
