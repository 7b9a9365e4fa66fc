// Internal declarations shared by the C ABI (stq_abi.cpp) and the kernels
// (stq_kernels.cu). Not part of the public interface.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

struct stq_pool;

namespace stq {

constexpr int D = 128;           // d_k = d_v
constexpr int PIVOT = 16;        // width marker of an FP16 pivot unit
constexpr int SCHEME_STEPQUANT = 0;    // dual-axis refit
constexpr int SCHEME_ROW_ABSMAX = 1;   // symmetric per-key-row absmax baseline

// Error bits written by kernels into the pool's device error word.
constexpr uint32_t ERR_SLOT_RANGE = 1u;   // a slot index was outside [0, n_slots)
// Checked builds only (compiled with STQ_CHECKS): the decode step and the dequantiser
// also record
constexpr uint32_t ERR_CODE = 2u;         //   a stored code 0, which the quantiser never
                                          //   writes (an uninitialised or corrupted slot)
constexpr uint32_t ERR_NONFINITE = 4u;    //   a NaN or infinity in the updated state

// Device view of a pool: caller-owned state buffers plus the metadata the library
// uploaded into the caller-owned meta buffer. Passed to kernels by value.
struct PoolDev {
  int kind;                 // 0 = GDN, 1 = KDA
  int n_slots;
  int H;
  int n_pivot_rows;         // pivot rows per slot
  int max_head_bytes;       // largest per-head code + pivot bytes (staging size)
  uint64_t slot_code_bytes;
  uint8_t* codes;           // [n_slots, slot_code_bytes]
  void* scales;             // [n_slots, H, 2, D] float32, or binary16 if scale16
  uint16_t* pivots;         // [n_slots, n_pivot_rows, D] float16 bits
  // metadata (device)
  const uint32_t* head_code_off;    // [H] byte offset of head h's codes in a slot
  const uint32_t* head_code_bytes;  // [H]
  const uint32_t* head_piv_first;   // [H] index of head h's first pivot row in a slot
  const uint32_t* head_piv_count;   // [H]
  const uint32_t* head_bits;        // [H] the width shared by all rows of head h
                                    //   (2/4/6/8, or 16 if all rows are pivots), 0 if mixed
  const uint32_t* warp_code_off;    // [H*8] byte offset in head h where rows 16w.. start
  const uint4* warp_rec;            // [H*8] what the decode step prefetches for warp w of
                                    //   head h: {x: byte offset of head h in a slot,
                                    //   y: byte offset of rows 16w.. in head h, z: their
                                    //   code bytes, w: head width (low 8 bits, 0 if mixed)
                                    //   | index of the head's first pivot row << 8}
  const uint32_t* row_info;         // [H*D] bits (low 8) | byte offset in head << 8
                                    //   (pivot rows: index in head's pivot block << 8)
  const float* g;                   // [H*D] row gain (omega_i / mean omega)^(-1/2)
  const float* omega;               // [H*D]
  uint32_t* err;                    // [4] sticky error bits
  int scheme;                       // SCHEME_STEPQUANT or SCHEME_ROW_ABSMAX
  int any_mixed;                    // 1 if some head's rows have different widths
  int scale16;                      // 1: r and c stored as binary16
};

// Byte layout of the meta buffer, computed on the host.
struct MetaLayout {
  size_t head_code_off, head_code_bytes, head_piv_first, head_piv_count, head_bits;
  size_t warp_code_off, warp_rec, row_info, g, omega, err, total;
};

MetaLayout meta_layout(int H);

// Launchers (stq_kernels.cu). They return the cudaGetLastError() of the launch (or of
// the one-time set-up of the kernel's shared-memory size and the device's SM count).
cudaError_t launch_decode(const PoolDev& P, const int32_t* slots, int B, const float* q,
                          const float* k, const float* v, const float* gate,
                          const float* beta, float* out, cudaStream_t s);
cudaError_t launch_quantize(const PoolDev& P, const int32_t* slots, int B, const float* S,
                            cudaStream_t s);
cudaError_t launch_dequantize(const PoolDev& P, const int32_t* slots, int B, float* S_out,
                              cudaStream_t s);
// The same two steps with the per-key-row absmax quantiser (stq_absmax.cu);
// launch_decode / launch_quantize forward to them for a SCHEME_ROW_ABSMAX pool.
cudaError_t launch_decode_absmax(const PoolDev& P, const int32_t* slots, int B, const float* q,
                                 const float* k, const float* v, const float* gate,
                                 const float* beta, float* out, cudaStream_t s);
cudaError_t launch_quantize_absmax(const PoolDev& P, const int32_t* slots, int B, const float* S,
                                   cudaStream_t s);
cudaError_t launch_fp32_step(int kind, int B, int H, float* S, const float* q,
                             const float* k, const float* v, const float* gate,
                             const float* beta, float* out, cudaStream_t s);

// Device staging of one host-buffer decode step for B requests: q, k, v, gate, beta and
// the readout, each 16-byte aligned (byte offsets; element counts). Used by
// stq_decode_step_host, stq_decode_step_host_static and the pipeline (stq_abi.cpp).
struct StagingLayout {
  size_t q, k, v, gate, beta, out, total;
  size_t n_vec, n_gate, n_beta;
};
StagingLayout staging_layout(const PoolDev& P, int B);

// The argument checks every batched entry point makes (pool not NULL, 0 <= B,
// B * H < 2^31, d_slots not NULL when B > 0). Returns an stq_status (0 = STQ_OK) and
// sets the thread's last error message on failure.
int check_batch(const struct ::stq_pool* pool, const int32_t* d_slots, int B);

// Accessors for entry points that live outside stq_abi.cpp.
const PoolDev* pool_dev(const struct ::stq_pool* pool);
int pool_kind(const struct ::stq_pool* pool);
void set_last_error(const char* msg);
void clear_last_error();

}  // namespace stq
