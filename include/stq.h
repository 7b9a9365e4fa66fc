/*
 * stq.h -- C ABI of the B200 packed Delta-rule state decode step.
 *
 * The operation is the per-(request, head) decode step over a low-bit recurrent
 * state from "STEPQuant: When and Where Errors Matter in Delta-Rule Recurrent State
 * Quantization" (arXiv 2609.38169), as these web pages describe it:
 *   - gated delta rule S_t = (I - beta_t k_t k_t^T) D_t S_{t-1} + beta_t k_t v_t^T,
 *     D_t a per-head scalar alpha_t (Gated DeltaNet, "GDN") or a per-key-channel
 *     diagonal (Kimi Delta Attention, "KDA")  [bloombook.cn tutorial, section 2];
 *   - readout o_t = S_t^T q_t from the updated floating-point state, then
 *     requantise and store, so this step's error only reaches later steps
 *     [singularity-lens.com summary, decode-order paragraph];
 *   - dual-axis codes X_ij = r_i c_j z_ij with a key-row scale r_i and a value-column
 *     scale c_j fitted under omega-weighted squared error  [bloombook section 4;
 *     singularity-lens dual-axis paragraph];
 *   - per-unit widths (unit = head for GDN, key row for KDA) from {2,4,6,8} and FP16
 *     pivot units kept unquantised, fixed offline for all requests  [ai-trend.me
 *     review, Method; singularity-lens calibration paragraph].
 * The exact float32 evaluation order (tree sums, where the decay is folded, the
 * refit rule) is the one the CPU oracle restates; both sides follow it.
 *
 * Conventions for every call:
 *   - d_k = d_v = d = 128.
 *   - Pointers named d_* are device pointers; h_* are host pointers. Every device
 *     pointer must be 16-byte aligned (else STQ_ERR_ALIGNMENT).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls only enqueue work: the status covers argument checks and launch errors.
 *   - The caller owns every buffer. The library never allocates device memory; the
 *     pool handle owns only host memory (freed by stq_pool_destroy).
 *   - Kernels check slot indices against n_slots; a bad index sets a sticky error
 *     bit in the pool's device metadata and that (request, head) is skipped.
 *     stq_pool_check() reads and clears it. A checked build of the library (compiled
 *     with STQ_CHECKS; stq_version() then says "checked") also records stored codes 0
 *     (never written by the quantiser: an uninitialised or corrupted slot) and
 *     non-finite updated states; those heads are still processed.
 *   - No call may list the same slot twice in one batch.
 *   - Stream capture: stq_decode_step, stq_quantize_init, stq_dequantize,
 *     stq_decode_step_host, stq_row_sq_error and stq_row_error_at_widths only enqueue
 *     work on `stream` (no allocation, no synchronisation), so they can be recorded
 *     into a CUDA graph. Make the first call of stq_decode_step (or of a call that runs
 *     it), stq_quantize_init, stq_dequantize and stq_decode_step_host_static on a device
 *     outside capture: each sets itself up once per device (a kernel's shared-memory
 *     limit, the number of CTAs the device holds at once, the static staging address).
 *     stq_pool_check and the pipeline calls synchronise and cannot be captured.
 *   - Errors: a non-zero stq_status; stq_last_error() gives a message (thread-local).
 *   - No C++ exception crosses this boundary.
 */
#ifndef STQ_H
#define STQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  STQ_OK = 0,
  STQ_ERR_INVALID_ARG = 1,   /* a size, kind, width or pointer is invalid */
  STQ_ERR_ALIGNMENT = 2,     /* a device pointer is not 16-byte aligned */
  STQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  STQ_ERR_DEVICE_CHECK = 4   /* a kernel recorded a device check (stq_pool_check) */
} stq_status;

typedef enum { STQ_GDN = 0, STQ_KDA = 1 } stq_kind;

/* How a decode step (and stq_quantize_init) requantises the updated state.
 *   STQ_SCHEME_STEPQUANT: the dual-axis refit r_i c_j z_ij of the method (row scale from
 *     the row's mean magnitude and influence, column scale from two omega-weighted
 *     least-squares steps)  [bloombook section 4; singularity-lens dual-axis paragraph].
 *   STQ_SCHEME_ROW_ABSMAX: the pages' uniform comparison quantiser, symmetric per-key-row
 *     absmax: r_i = max_j |S_ij| * fl(1/qmax_i), codes rint(S_ij * fl(1/r_i)), all column
 *     scales 1  [singularity-lens calibration and evaluation-setup paragraphs].
 * Both keep the same pool layout, widths and FP16 pivot units. */
typedef enum { STQ_SCHEME_STEPQUANT = 0, STQ_SCHEME_ROW_ABSMAX = 1 } stq_scheme;

#define STQ_D 128
#define STQ_PIVOT_BITS 16

/* Static description of a state pool: the per-unit widths and row influences are
 * fixed offline and shared by every request (ai-trend review, Method (1)). */
typedef struct {
  int kind;                  /* stq_kind */
  int n_slots;               /* number of state slots, > 0 */
  int H;                     /* heads per slot, > 0 */
  int d;                     /* must be STQ_D */
  const uint8_t* unit_bits;  /* host; GDN: [H] (one width per head), KDA: [H*d]
                                (one width per key row); each 2, 4, 6, 8 or 16 (FP16
                                pivot unit) */
  const float* omega;        /* host; [H*d] row influence omega_i, finite and > 0 */
  int scheme;                /* stq_scheme; 0 (zero-initialised) = STQ_SCHEME_STEPQUANT */
  int scale_bits;            /* storage of r and c: 32 (float32; 0 means 32) or 16
                                (IEEE binary16, the compact layout: r is rounded to
                                binary16 when formed, the final c before the codes are
                                fitted to it, so the stored triple stays consistent) */
} stq_pool_desc;

/* Buffer sizes (bytes) the caller allocates for a pool, from stq_pool_layout. */
typedef struct {
  size_t codes_bytes;        /* packed codes, all slots */
  size_t scales_bytes;       /* r[d], c[d] per (slot, head), float32 or binary16 */
  size_t pivots_bytes;       /* float16 pivot rows, all slots */
  size_t meta_bytes;         /* device metadata the library writes at create time */
  size_t slot_code_bytes;    /* bytes of packed codes per slot */
  int n_pivot_rows;          /* pivot rows per slot */
  int max_head_bytes;        /* largest per-head code + pivot bytes */
} stq_pool_sizes;

typedef struct stq_pool stq_pool;

/* Layout of one pool, host only (no CUDA call). Slot s holds, for head h, the rows
 * of its non-pivot units back to back (row i of width b takes 16*b bytes; code j of a
 * row is bits [b*j, b*j+b) of a little-endian bit stream, stored as
 * u = Q + 2^(b-1)); the float16 rows of its pivot units in (head, row) order; and
 * r[128], c[128] per head (float32, or binary16 when scale_bits is 16). Returns
 * STQ_ERR_INVALID_ARG on a bad description. The pages fix what is stored -- integer
 * codes of the unit's width times a row and a column scale, pivot units in FP16
 * (bloombook section 4; ai-trend review, Method) -- and that a slot serves one request
 * (zhichai forum reply: five slots per request); the byte layout is this library's. */
stq_status stq_pool_layout(const stq_pool_desc* desc, stq_pool_sizes* out);

/* Bind caller-allocated device buffers (sizes from stq_pool_layout) to a new pool
 * handle and upload the static metadata (offsets, widths, omega_i and the row gain
 * g_i = (omega_i / mean omega)^(-1/2)) into d_meta with a synchronous copy. The
 * state buffers are not touched: fill them with stq_quantize_init. d_pivots may be
 * NULL when the pool has no pivot rows. The widths and row influences are fixed once
 * for all requests (ai-trend review, Method (1); singularity-lens calibration
 * paragraph); the row gain is the omega_i^(-1/2) factor of the row scale (bloombook
 * section 4). Errors: STQ_ERR_INVALID_ARG (description, NULL buffers),
 * STQ_ERR_ALIGNMENT, STQ_ERR_CUDA (the metadata copy). */
stq_status stq_pool_create(const stq_pool_desc* desc, void* d_codes, void* d_scales,
                           void* d_pivots, void* d_meta, stq_pool** out);

/* Free the host handle. Device buffers stay the caller's. NULL is ignored. */
void stq_pool_destroy(stq_pool* pool);

/* Quantise float32 states into the pool: for b < B, slot d_slots[b] receives
 * d_S[b] ([H, 128, 128], row-major, key row i, value column j) under the refit rule
 * (row scale, column scale start, two omega-weighted least-squares steps, final
 * codes; bloombook section 4). Pivot units store float16(S). */
stq_status stq_quantize_init(stq_pool* pool, const int32_t* d_slots, int B,
                             const float* d_S, void* stream);

/* One decode step for B requests (THE hot path; the fused decode kernel of bloombook
 * section 4 and the decode order of the singularity-lens summary). For request b and
 * head h, with slot s = d_slots[b]:
 *   restore S' = D_t * dequantised state of (s, h), update with the gated delta rule,
 *   write out[b, h, :] = S_t^T q (float32, from the updated unquantised state), refit
 *   the scales and store S_t back into slot s packed.
 * q, k, v: [B, H, 128] float32 device. gate: GDN [B, H] retention alpha_t, KDA
 * [B, H, 128] per-key-row retention; values in [0, 1] (the host takes exp of the
 * log-retention). beta: [B, H] in [0, 1]. out: [B, H, 128] float32 device. */
stq_status stq_decode_step(stq_pool* pool, const int32_t* d_slots, int B,
                           const float* d_q, const float* d_k, const float* d_v,
                           const float* d_gate, const float* d_beta, float* d_out,
                           void* stream);

/* Bytes of device staging stq_decode_step_host needs for B requests. */
size_t stq_decode_step_host_staging_bytes(const stq_pool* pool, int B);

/* The same decode step with its per-step inputs and output in HOST memory (pinned
 * for asynchronous copies): copies h_q, h_k, h_v, h_gate, h_beta into d_staging,
 * runs stq_decode_step, and copies the output back into h_out, all on `stream`.
 * d_slots stays a device array. The caller synchronises the stream before reading
 * h_out. staging_bytes must be >= stq_decode_step_host_staging_bytes(pool, B). */
stq_status stq_decode_step_host(stq_pool* pool, const int32_t* d_slots, int B,
                                const float* h_q, const float* h_k, const float* h_v,
                                const float* h_gate, const float* h_beta, float* h_out,
                                void* d_staging, size_t staging_bytes, void* stream);

/* ---- The host-buffer step pipelined inside the library ---------------------------
 * A serving loop that keeps its per-step inputs and outputs in host memory overlaps
 * the copies with the decode: step i's inputs go up on the pipeline's upload stream
 * while step i-1 decodes, and step i's readout comes down on its download stream while
 * step i+1 decodes. The decode steps stay in order on the caller's stream, as the
 * decode-order paragraph of the singularity-lens.com summary requires (each step reads
 * the state the previous one wrote). The pipeline owns two CUDA streams and eight
 * events (created by stq_pipeline_create, released by stq_pipeline_destroy) and no
 * device memory: two halves of the caller's staging buffer alternate between steps. */
typedef struct stq_pipeline stq_pipeline;

/* Bytes of device staging a pipeline of B requests needs (two halves, each holding
 * one step's q, k, v, gate, beta and readout); 0 for a NULL pool or B < 0. */
size_t stq_pipeline_staging_bytes(const stq_pool* pool, int B);

/* A pipeline for steps of B > 0 requests of `pool`, on the current device (make every
 * later call on it with that device current). d_staging: caller-owned device buffer of
 * staging_bytes >= stq_pipeline_staging_bytes(pool, B), 16-byte aligned, that the
 * pipeline uses until stq_pipeline_destroy. Errors: STQ_ERR_INVALID_ARG (sizes, NULL),
 * STQ_ERR_ALIGNMENT, STQ_ERR_CUDA (stream or event creation). */
stq_status stq_pipeline_create(stq_pool* pool, int B, void* d_staging, size_t staging_bytes,
                               stq_pipeline** out);

/* Enqueue one decode step (stq_decode_step's operation; q, k, v, gate, beta and out
 * have its shapes, in host memory, pinned for the copies to overlap): the inputs are
 * copied up on the upload stream, the step runs on `stream`, its readout is copied
 * into h_out on the download stream. Then the call waits on the host until the
 * PREVIOUS call's readout is in that call's h_out, and returns. So on return the
 * previous step's h_out is complete, and the host inputs and h_out of the step before
 * it may be reused. d_slots (device, B entries) must stay unchanged until the step's
 * decode has run. */
stq_status stq_pipeline_step(stq_pipeline* pipe, const int32_t* d_slots, const float* h_q,
                             const float* h_k, const float* h_v, const float* h_gate,
                             const float* h_beta, float* h_out, void* stream);

/* Wait on the host for the last step's readout, and make `stream` wait for it too
 * (work enqueued on `stream` afterwards follows every pipelined copy). */
stq_status stq_pipeline_finish(stq_pipeline* pipe, void* stream);

/* Synchronise the pipeline's streams and release them and its events. NULL is
 * ignored. The staging buffer stays the caller's. */
void stq_pipeline_destroy(stq_pipeline* pipe);

/* Bytes of the library's own device staging array used by
 * stq_decode_step_host_static (8 MiB). */
#define STQ_STATIC_STAGING_BYTES (8u << 20)

/* stq_decode_step_host without a caller-provided staging buffer. The paper has no
 * counterpart: this is a service of this library for callers that cannot allocate
 * device memory on their decode path -- a host application that was handed the state
 * pool once and only has host buffers per step, or a serving loop that must not take
 * the device-wide synchronisation a cudaMalloc implies. The per-step device staging
 * (q, k, v, gate, beta and the readout) lives in a fixed array of
 * STQ_STATIC_STAGING_BYTES that the library declares in device memory; every GPU that
 * loads the library holds it until the process exits. Arguments are those of
 * stq_decode_step_host minus d_staging/staging_bytes.
 *   - Returns STQ_ERR_INVALID_ARG (with a message) when the step's staging for B
 *     requests exceeds STQ_STATIC_STAGING_BYTES (about 3,200 KDA or 4,000 GDN
 *     head-states per call); use stq_decode_step_host with your own buffer then.
 *   - Calls no cudaMalloc/cudaFree and no allocating routine.
 *   - The first call on each device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture on the device. The address is kept per device ordinal for the life of
 *     the process: it belongs to the device's primary context, so do not call this
 *     entry point after cudaDeviceReset on that device, nor with a context other than
 *     the primary one current (use stq_decode_step_host then).
 *   - All calls share the one array, which keeps the last call's contents (nothing in
 *     it needs to start at zero: each call writes every byte it reads). Calls whose
 *     work overlaps on the GPU (other streams, other host threads) race on it: order
 *     them on one stream or synchronise between them. */
stq_status stq_decode_step_host_static(stq_pool* pool, const int32_t* d_slots, int B,
                                       const float* h_q, const float* h_k, const float* h_v,
                                       const float* h_gate, const float* h_beta, float* h_out,
                                       void* stream);

/* Dequantise slots d_slots[0..B) into d_S_out [B, H, 128, 128] float32:
 * S_ij = (Q_ij * r_i) * c_j, pivot rows float32(h_ij) -- the restored state
 * X_ij = r_i c_j z_ij of bloombook section 4, without the decay of a step. Errors as
 * stq_decode_step; the first call on a device raises the kernel's shared-memory limit
 * (make it outside stream capture). */
stq_status stq_dequantize(stq_pool* pool, const int32_t* d_slots, int B, float* d_S_out,
                          void* stream);

/* FP32-state decode step (the unquantised state the pages compare against), in place
 * on d_S [B, H, 128, 128]: S <- (I - beta k k^T) D S + beta k v^T, out = S^T q.
 * Same inputs as stq_decode_step; kind selects the gate shape. */
stq_status stq_fp32_decode_step(int kind, int B, int H, int d, float* d_S,
                                const float* d_q, const float* d_k, const float* d_v,
                                const float* d_gate, const float* d_beta, float* d_out,
                                void* stream);

/* ---- Offline calibration: the lifetime-aware width allocation that fixes a pool's
 * unit_bits before any decode step (bloombook section 3, lifetime weight, and section 4,
 * "time" half: budgeted allocation and FP16 pivots; singularity-lens calibration
 * paragraph: distortion per candidate width, candidates {2,4,6,8} or {4,6,8}). The
 * per-width distortions come from the calibration states quantised with
 * stq_quantize_init into a pool of one uniform width and read back with
 * stq_dequantize; stq_row_sq_error measures them. ---------------------------------- */

/* Per-row squared error of n_states 128x128 float32 states against their
 * reconstructions: e[s*128 + i] (+)= sum_j (S[s,i,j] - S_hat[s,i,j])^2, the squares of
 * the float32 differences summed as a balanced binary tree over j. accumulate != 0 adds
 * to d_err (float32, one rounding) instead of overwriting it. Device pointers, 16-byte
 * aligned; n_states >= 0. Enqueued on `stream`. */
stq_status stq_row_sq_error(const float* d_S, const float* d_S_hat, int n_states, float* d_err,
                            int accumulate, void* stream);

/* In-head distortion of every row at candidate widths, for the allocation of per-row
 * widths (KDA): the rows of a head share the column scales c_j, so a row's width only
 * sets how far its codes reach. For b < B, head h, row i and candidate k, with
 * S = d_S[b] ([H, 128, 128] float32) and c the column scales stored in slot
 * d_slots[b] (fill the slot with stq_quantize_init of the same states first):
 *   r_i = the refit's row scale of S's row i (computed for every row, pivot rows too;
 *         rounded to binary16 in a compact pool, as the refit stores it),
 *   Q_ij = clamp(rint((S_ij * fl(1/r_i)) * fl(1/c_j)), +-(2^(b_k-1) - 1)),
 *   d_err[((b H + h) 128 + i) n_cand + k] = tree sum_j (S_ij - (Q_ij r_i) c_j)^2
 * (the tree of stq_row_sq_error). h_cand_bits: 1 to 4 widths from {2,4,6,8} (host).
 * At a row's own width this is the row's error in the quantised slot. Device pointers
 * 16-byte aligned; enqueued on `stream`; a slot outside the pool is flagged as in
 * stq_decode_step. (bloombook section 4, budgeted allocation; singularity-lens
 * calibration paragraph: per-row squared error for KDA units.) */
stq_status stq_row_error_at_widths(stq_pool* pool, const int32_t* d_slots, int B, const float* d_S,
                                   const int* h_cand_bits, int n_cand, float* d_err, void* stream);

/* Lifetime weights L_u = sum_{j=0}^{horizon-1} exp(2 j ell_u) of n units, ell_u the
 * unit's mean log-retention (<= 0), summed term by term in double. Host arrays. */
stq_status stq_lifetime_weights(const double* ell, int n, int horizon, double* out);

/* Distortion of each unit from the row errors of N calibration states
 * (h_row_err [N, H, 128], from stq_row_sq_error of states quantised at one width):
 * GDN (kind 0) one value per head, sum_n sum_i omega_i e[n,h,i] / (N 128^2);
 * KDA (kind 1) one value per key row (h, i), sum_n e[n,h,i] / (N 128).
 * Sequential double sums (n outer, i inner). Host arrays; out has H (GDN) or H*128
 * (KDA) entries. */
stq_status stq_unit_distortion(int kind, int N, int H, const float* h_row_err,
                               const float* h_omega, double* out);

/* Widths for n units: the n_pivots units with the largest lifetime[u] * dist[u, last]
 * (ties: lower index) get STQ_PIVOT_BITS; the others minimise
 * sum_u lifetime[u] * dist[u, c_u] subject to sum_u cand_bits[c_u] <= budget * (their
 * count), solved exactly (dynamic program over the total width; among equal costs the
 * narrower width, then the smaller total). cand_bits: n_cand ascending even widths from
 * {2,4,6,8}; dist [n, n_cand] row-major. Returns STQ_ERR_INVALID_ARG for an infeasible
 * budget or bad candidates. Host arrays; the result goes to out_bits [n]. */
stq_status stq_allocate_bits(int n, int n_cand, const int* cand_bits, const double* lifetime,
                             const double* dist, double budget, int n_pivots, uint8_t* out_bits);

/* Issue-rate probe (a measurement aid with no counterpart in the pages): launches
 * `blocks` CTAs of 512 threads on `stream`; each thread runs 8 independent
 * register-only chains of `iters` instructions of one kind -- mode 0: packed
 * fma.rn.f32x2 (2 lane operations each), 1: scalar fma.rn.f32, 2: lop3.b32 -- and
 * writes one float per thread to d_out (device, blocks * 512 floats, caller-owned).
 * Timed by the caller with CUDA events it gives the rate at which the GPU retires that
 * instruction kind: blocks * 512 * 8 * iters lane operations (twice that for mode 0).
 * The decode step is bound by instruction issue on the CUDA cores; this is the measured
 * rate its roofline is read against. Errors: STQ_ERR_INVALID_ARG (mode, blocks outside
 * [1, 65535], iters < 1, NULL d_out), STQ_ERR_CUDA (launch). */
stq_status stq_issue_rate_probe(int mode, int blocks, int iters, float* d_out, void* stream);

/* Synchronise `stream`, read the pool's sticky device error bits, clear them, and
 * return STQ_ERR_DEVICE_CHECK if any was set (message names the check). */
stq_status stq_pool_check(stq_pool* pool, void* stream);

/* Message of the last failing call on this thread ("" if none). */
const char* stq_last_error(void);

/* Library version string. */
const char* stq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STQ_H */
