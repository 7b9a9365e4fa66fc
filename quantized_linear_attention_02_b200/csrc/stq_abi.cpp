// C ABI of the packed Delta-rule state decode step: argument checks, pool layout,
// metadata upload and kernel launches. See include/stq.h for the contract.
#include "stq.h"

#include <cmath>
#include <cstdarg>
#include <initializer_list>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "stq_internal.h"

namespace {

thread_local std::string g_last_error;

stq_status fail(stq_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
stq_status fail(stq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

stq_status ok() {
  g_last_error.clear();
  return STQ_OK;
}

stq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(STQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t up16(size_t x) { return (x + 15) & ~size_t(15); }

// Host-side layout of one pool, derived from the description.
struct HostLayout {
  int kind = 0, n_slots = 0, H = 0, scheme = 0, scale_bytes = 4;
  std::vector<uint32_t> head_code_off, head_code_bytes, head_piv_first, head_piv_count, head_bits;
  std::vector<uint32_t> warp_code_off;
  std::vector<uint32_t> row_info;
  std::vector<float> g, omega;
  uint64_t slot_code_bytes = 0;
  int n_pivot_rows = 0;
  int max_head_bytes = 0;
};

stq_status build_layout(const stq_pool_desc* desc, HostLayout& L) {
  if (desc == nullptr) return fail(STQ_ERR_INVALID_ARG, "desc is NULL");
  if (desc->kind != STQ_GDN && desc->kind != STQ_KDA)
    return fail(STQ_ERR_INVALID_ARG, "kind must be STQ_GDN (0) or STQ_KDA (1), got %d", desc->kind);
  if (desc->d != STQ_D) return fail(STQ_ERR_INVALID_ARG, "d must be %d, got %d", STQ_D, desc->d);
  if (desc->scheme != STQ_SCHEME_STEPQUANT && desc->scheme != STQ_SCHEME_ROW_ABSMAX)
    return fail(STQ_ERR_INVALID_ARG,
                "scheme must be STQ_SCHEME_STEPQUANT (0) or STQ_SCHEME_ROW_ABSMAX (1), got %d", desc->scheme);
  if (desc->n_slots <= 0) return fail(STQ_ERR_INVALID_ARG, "n_slots must be > 0, got %d", desc->n_slots);
  if (desc->H <= 0 || desc->H > (1 << 20)) return fail(STQ_ERR_INVALID_ARG, "H out of range: %d", desc->H);
  if (desc->unit_bits == nullptr || desc->omega == nullptr)
    return fail(STQ_ERR_INVALID_ARG, "unit_bits and omega must be non-NULL host arrays");
  const int H = desc->H, D = STQ_D;
  L.kind = desc->kind;
  L.scheme = desc->scheme;
  if (desc->scale_bits != 0 && desc->scale_bits != 32 && desc->scale_bits != 16)
    return fail(STQ_ERR_INVALID_ARG, "scale_bits must be 16 or 32 (0 = 32), got %d", desc->scale_bits);
  L.scale_bytes = desc->scale_bits == 16 ? 2 : 4;
  L.n_slots = desc->n_slots;
  L.H = H;
  L.head_code_off.assign(H, 0);
  L.head_code_bytes.assign(H, 0);
  L.head_piv_first.assign(H, 0);
  L.head_piv_count.assign(H, 0);
  L.head_bits.assign(H, 0);
  L.row_info.assign(size_t(H) * D, 0);
  L.warp_code_off.assign(size_t(H) * 8, 0);
  L.g.assign(size_t(H) * D, 0.0f);
  L.omega.assign(size_t(H) * D, 0.0f);
  uint64_t off = 0;
  int piv = 0;
  for (int h = 0; h < H; ++h) {
    L.head_code_off[h] = uint32_t(off);
    L.head_piv_first[h] = uint32_t(piv);
    uint32_t in_head = 0, piv_in_head = 0;
    double acc = 0.0;
    for (int i = 0; i < D; ++i) {
      const float om = desc->omega[size_t(h) * D + i];
      if (!(std::isfinite(om) && om > 0.0f))
        return fail(STQ_ERR_INVALID_ARG, "omega[%d][%d] must be finite and > 0", h, i);
      L.omega[size_t(h) * D + i] = om;
      acc += double(om);
    }
    // g_i = (omega_i / mean omega)^(-1/2): sequential float64 sum, divide, sqrt, reciprocal
    const double mean = acc / D;
    for (int i = 0; i < D; ++i) {
      const double wi = double(L.omega[size_t(h) * D + i]);
      L.g[size_t(h) * D + i] = float(1.0 / std::sqrt(wi / mean));
    }
    for (int i = 0; i < D; ++i) {
      const int b = (desc->kind == STQ_GDN) ? desc->unit_bits[h] : desc->unit_bits[size_t(h) * D + i];
      if (b != 2 && b != 4 && b != 6 && b != 8 && b != STQ_PIVOT_BITS)
        return fail(STQ_ERR_INVALID_ARG, "unit width %d (head %d row %d) not in {2,4,6,8,16}", b, h, i);
      if (i % 16 == 0) L.warp_code_off[size_t(h) * 8 + i / 16] = in_head;
      if (b == STQ_PIVOT_BITS) {
        L.row_info[size_t(h) * D + i] = uint32_t(b) | (piv_in_head << 8);
        ++piv_in_head;
      } else {
        L.row_info[size_t(h) * D + i] = uint32_t(b) | (in_head << 8);
        in_head += uint32_t(D * b / 8);
      }
    }
    uint32_t hb0 = L.row_info[size_t(h) * D] & 0xFFu;
    for (int i = 1; i < D; ++i)
      if ((L.row_info[size_t(h) * D + i] & 0xFFu) != hb0) hb0 = 0;
    L.head_bits[h] = hb0;
    L.head_code_bytes[h] = in_head;
    L.head_piv_count[h] = piv_in_head;
    off += in_head;
    piv += int(piv_in_head);
    const int hb = int(in_head + piv_in_head * D * 2);
    if (hb > L.max_head_bytes) L.max_head_bytes = hb;
  }
  if (off > 0xFFFFFFFFull)
    return fail(STQ_ERR_INVALID_ARG, "packed codes of one slot exceed 4 GiB (%llu bytes)",
                static_cast<unsigned long long>(off));
  if (piv >= (1 << 24))
    return fail(STQ_ERR_INVALID_ARG, "too many FP16 pivot rows per slot: %d (limit %d)", piv, (1 << 24) - 1);
  L.slot_code_bytes = off;
  L.n_pivot_rows = piv;
  return STQ_OK;
}

}  // namespace

namespace stq {

MetaLayout meta_layout(int H) {
  MetaLayout m;
  size_t o = 0;
  m.head_code_off = o;   o = up16(o + size_t(H) * 4);
  m.head_code_bytes = o; o = up16(o + size_t(H) * 4);
  m.head_piv_first = o;  o = up16(o + size_t(H) * 4);
  m.head_piv_count = o;  o = up16(o + size_t(H) * 4);
  m.head_bits = o;       o = up16(o + size_t(H) * 4);
  m.warp_code_off = o;   o = up16(o + size_t(H) * 8 * 4);
  m.warp_rec = o;        o = up16(o + size_t(H) * 8 * 16);
  m.row_info = o;        o = up16(o + size_t(H) * D * 4);
  m.g = o;               o = up16(o + size_t(H) * D * 4);
  m.omega = o;           o = up16(o + size_t(H) * D * 4);
  m.err = o;             o = up16(o + 16);
  m.total = o;
  return m;
}

}  // namespace stq

struct stq_pool {
  HostLayout L;
  stq::PoolDev dev;
  void* meta = nullptr;
};

namespace stq {

const PoolDev* pool_dev(const ::stq_pool* pool) { return pool ? &pool->dev : nullptr; }
int pool_kind(const ::stq_pool* pool) { return pool ? pool->L.kind : -1; }
void set_last_error(const char* msg) { g_last_error = msg; }
void clear_last_error() { g_last_error.clear(); }

}  // namespace stq

extern "C" {

const char* stq_last_error(void) { return g_last_error.c_str(); }

#ifdef STQ_CHECKS
const char* stq_version(void) { return "stq 0.1 (sm_100a, checked)"; }
#else
const char* stq_version(void) { return "stq 0.1 (sm_100a)"; }
#endif

stq_status stq_pool_layout(const stq_pool_desc* desc, stq_pool_sizes* out) {
  if (out == nullptr) return fail(STQ_ERR_INVALID_ARG, "out is NULL");
  HostLayout L;
  stq_status st = build_layout(desc, L);
  if (st != STQ_OK) return st;
  const size_t ns = size_t(desc->n_slots);
  out->slot_code_bytes = size_t(L.slot_code_bytes);
  out->codes_bytes = ns * size_t(L.slot_code_bytes);
  out->scales_bytes = ns * size_t(L.H) * 2 * STQ_D * size_t(L.scale_bytes);
  out->pivots_bytes = ns * size_t(L.n_pivot_rows) * STQ_D * 2;
  out->meta_bytes = stq::meta_layout(L.H).total;
  out->n_pivot_rows = L.n_pivot_rows;
  out->max_head_bytes = L.max_head_bytes;
  return ok();
}

stq_status stq_pool_create(const stq_pool_desc* desc, void* d_codes, void* d_scales,
                           void* d_pivots, void* d_meta, stq_pool** out) {
  if (out == nullptr) return fail(STQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  stq_pool* p = new (std::nothrow) stq_pool();
  if (p == nullptr) return fail(STQ_ERR_INVALID_ARG, "out of host memory");
  stq_status st = build_layout(desc, p->L);
  if (st != STQ_OK) { delete p; return st; }
  const HostLayout& L = p->L;
  if (d_codes == nullptr || d_scales == nullptr || d_meta == nullptr ||
      (L.n_pivot_rows > 0 && d_pivots == nullptr)) {
    delete p;
    return fail(STQ_ERR_INVALID_ARG, "a device buffer is NULL");
  }
  if (!aligned16(d_codes) || !aligned16(d_scales) || !aligned16(d_meta) ||
      (d_pivots != nullptr && !aligned16(d_pivots))) {
    delete p;
    return fail(STQ_ERR_ALIGNMENT, "device buffers must be 16-byte aligned");
  }
  const stq::MetaLayout m = stq::meta_layout(L.H);
  std::vector<uint8_t> host(m.total, 0);
  auto put = [&](size_t at, const void* src, size_t n) { std::memcpy(host.data() + at, src, n); };
  put(m.head_code_off, L.head_code_off.data(), L.H * 4);
  put(m.head_code_bytes, L.head_code_bytes.data(), L.H * 4);
  put(m.head_piv_first, L.head_piv_first.data(), L.H * 4);
  put(m.head_piv_count, L.head_piv_count.data(), L.H * 4);
  put(m.head_bits, L.head_bits.data(), L.H * 4);
  put(m.warp_code_off, L.warp_code_off.data(), L.warp_code_off.size() * 4);
  {
    std::vector<uint32_t> rec(size_t(L.H) * 8 * 4);
    for (int h = 0; h < L.H; ++h)
      for (int w = 0; w < 8; ++w) {
        const size_t hw = size_t(h) * 8 + w;
        const uint32_t end = (w + 1 < 8) ? L.warp_code_off[hw + 1] : L.head_code_bytes[h];
        rec[4 * hw + 0] = L.head_code_off[h];
        rec[4 * hw + 1] = L.warp_code_off[hw];
        rec[4 * hw + 2] = end - L.warp_code_off[hw];
        rec[4 * hw + 3] = L.head_bits[h] | (L.head_piv_first[h] << 8);
      }
    put(m.warp_rec, rec.data(), rec.size() * 4);
  }
  put(m.row_info, L.row_info.data(), L.row_info.size() * 4);
  put(m.g, L.g.data(), L.g.size() * 4);
  put(m.omega, L.omega.data(), L.omega.size() * 4);
  cudaError_t e = cudaMemcpy(d_meta, host.data(), m.total, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) { delete p; return cuda_fail(e, "upload of pool metadata"); }
  uint8_t* mb = static_cast<uint8_t*>(d_meta);
  stq::PoolDev& dv = p->dev;
  dv.kind = L.kind;
  dv.n_slots = L.n_slots;
  dv.H = L.H;
  dv.n_pivot_rows = L.n_pivot_rows;
  dv.max_head_bytes = L.max_head_bytes;
  dv.slot_code_bytes = L.slot_code_bytes;
  dv.codes = static_cast<uint8_t*>(d_codes);
  dv.scales = d_scales;
  dv.scale16 = L.scale_bytes == 2;
  dv.pivots = static_cast<uint16_t*>(d_pivots);
  dv.head_code_off = reinterpret_cast<const uint32_t*>(mb + m.head_code_off);
  dv.head_code_bytes = reinterpret_cast<const uint32_t*>(mb + m.head_code_bytes);
  dv.head_piv_first = reinterpret_cast<const uint32_t*>(mb + m.head_piv_first);
  dv.head_piv_count = reinterpret_cast<const uint32_t*>(mb + m.head_piv_count);
  dv.head_bits = reinterpret_cast<const uint32_t*>(mb + m.head_bits);
  dv.warp_code_off = reinterpret_cast<const uint32_t*>(mb + m.warp_code_off);
  dv.warp_rec = reinterpret_cast<const uint4*>(mb + m.warp_rec);
  dv.row_info = reinterpret_cast<const uint32_t*>(mb + m.row_info);
  dv.g = reinterpret_cast<const float*>(mb + m.g);
  dv.omega = reinterpret_cast<const float*>(mb + m.omega);
  dv.err = reinterpret_cast<uint32_t*>(mb + m.err);
  dv.scheme = L.scheme;
  dv.any_mixed = 0;
  for (int h = 0; h < L.H; ++h)
    if (L.head_bits[h] == 0) dv.any_mixed = 1;
  p->meta = d_meta;
  *out = p;
  return ok();
}

void stq_pool_destroy(stq_pool* pool) { delete pool; }

}  // extern "C"

namespace stq {

int check_batch(const ::stq_pool* pool, const int32_t* d_slots, int B) {
  if (pool == nullptr) return fail(STQ_ERR_INVALID_ARG, "pool is NULL");
  if (B < 0) return fail(STQ_ERR_INVALID_ARG, "B must be >= 0, got %d", B);
  if (int64_t(B) * pool->L.H > (int64_t(1) << 31) - 1)
    return fail(STQ_ERR_INVALID_ARG, "B * H too large: %d * %d", B, pool->L.H);
  if (B > 0 && d_slots == nullptr) return fail(STQ_ERR_INVALID_ARG, "d_slots is NULL");
  return STQ_OK;
}

StagingLayout staging_layout(const PoolDev& P, int B) {
  StagingLayout s;
  const size_t BH = size_t(B) * size_t(P.H);
  s.n_vec = BH * STQ_D;
  s.n_gate = (P.kind == STQ_GDN) ? BH : BH * STQ_D;
  s.n_beta = BH;
  size_t o = 0;
  s.q = o;    o = up16(o + s.n_vec * 4);
  s.k = o;    o = up16(o + s.n_vec * 4);
  s.v = o;    o = up16(o + s.n_vec * 4);
  s.gate = o; o = up16(o + s.n_gate * 4);
  s.beta = o; o = up16(o + s.n_beta * 4);
  s.out = o;  o = up16(o + s.n_vec * 4);
  s.total = o;
  return s;
}

}  // namespace stq

extern "C" {

static stq_status check_batch(const stq_pool* pool, const int32_t* d_slots, int B) {
  return static_cast<stq_status>(stq::check_batch(pool, d_slots, B));
}

static stq_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (p == nullptr) return fail(STQ_ERR_INVALID_ARG, "a device pointer is NULL");
    if (!aligned16(p)) return fail(STQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  }
  return STQ_OK;
}

stq_status stq_quantize_init(stq_pool* pool, const int32_t* d_slots, int B, const float* d_S,
                             void* stream) {
  stq_status st = check_batch(pool, d_slots, B);
  if (st != STQ_OK) return st;
  if (B == 0) return ok();
  st = check_ptrs({d_S});
  if (st != STQ_OK) return st;
  cudaError_t e = stq::launch_quantize(pool->dev, d_slots, B, d_S, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stq_quantize_init launch");
  return ok();
}

stq_status stq_decode_step(stq_pool* pool, const int32_t* d_slots, int B, const float* d_q,
                           const float* d_k, const float* d_v, const float* d_gate,
                           const float* d_beta, float* d_out, void* stream) {
  stq_status st = check_batch(pool, d_slots, B);
  if (st != STQ_OK) return st;
  if (B == 0) return ok();
  st = check_ptrs({d_q, d_k, d_v, d_gate, d_beta, d_out});
  if (st != STQ_OK) return st;
  cudaError_t e = stq::launch_decode(pool->dev, d_slots, B, d_q, d_k, d_v, d_gate, d_beta, d_out,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stq_decode_step launch");
  return ok();
}

size_t stq_decode_step_host_staging_bytes(const stq_pool* pool, int B) {
  if (pool == nullptr || B < 0) return 0;
  return stq::staging_layout(pool->dev, B).total;
}

stq_status stq_decode_step_host(stq_pool* pool, const int32_t* d_slots, int B, const float* h_q,
                                const float* h_k, const float* h_v, const float* h_gate,
                                const float* h_beta, float* h_out, void* d_staging,
                                size_t staging_bytes, void* stream) {
  stq_status st = check_batch(pool, d_slots, B);
  if (st != STQ_OK) return st;
  if (B == 0) return ok();
  if (!h_q || !h_k || !h_v || !h_gate || !h_beta || !h_out)
    return fail(STQ_ERR_INVALID_ARG, "a host pointer is NULL");
  st = check_ptrs({d_staging});
  if (st != STQ_OK) return st;
  const stq::StagingLayout L = stq::staging_layout(pool->dev, B);
  if (staging_bytes < L.total)
    return fail(STQ_ERR_INVALID_ARG, "staging_bytes %zu < required %zu", staging_bytes, L.total);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(d_staging);
  float* dq = reinterpret_cast<float*>(base + L.q);
  float* dk = reinterpret_cast<float*>(base + L.k);
  float* dvv = reinterpret_cast<float*>(base + L.v);
  float* dg = reinterpret_cast<float*>(base + L.gate);
  float* db = reinterpret_cast<float*>(base + L.beta);
  float* dout = reinterpret_cast<float*>(base + L.out);
  struct Copy { void* dst; const void* src; size_t n; };
  const Copy in[] = {{dq, h_q, L.n_vec * 4}, {dk, h_k, L.n_vec * 4}, {dvv, h_v, L.n_vec * 4},
                     {dg, h_gate, L.n_gate * 4}, {db, h_beta, L.n_beta * 4}};
  for (const Copy& c : in) {
    cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy of step inputs");
  }
  cudaError_t e = stq::launch_decode(pool->dev, d_slots, B, dq, dk, dvv, dg, db, dout, s);
  if (e != cudaSuccess) return cuda_fail(e, "stq_decode_step launch");
  e = cudaMemcpyAsync(h_out, dout, L.n_vec * 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy of the readout");
  return ok();
}

stq_status stq_dequantize(stq_pool* pool, const int32_t* d_slots, int B, float* d_S_out,
                          void* stream) {
  stq_status st = check_batch(pool, d_slots, B);
  if (st != STQ_OK) return st;
  if (B == 0) return ok();
  st = check_ptrs({d_S_out});
  if (st != STQ_OK) return st;
  cudaError_t e = stq::launch_dequantize(pool->dev, d_slots, B, d_S_out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stq_dequantize launch");
  return ok();
}

stq_status stq_fp32_decode_step(int kind, int B, int H, int d, float* d_S, const float* d_q,
                                const float* d_k, const float* d_v, const float* d_gate,
                                const float* d_beta, float* d_out, void* stream) {
  if (kind != STQ_GDN && kind != STQ_KDA) return fail(STQ_ERR_INVALID_ARG, "bad kind %d", kind);
  if (d != STQ_D) return fail(STQ_ERR_INVALID_ARG, "d must be %d, got %d", STQ_D, d);
  if (B < 0 || H <= 0 || int64_t(B) * H > (int64_t(1) << 31) - 1)
    return fail(STQ_ERR_INVALID_ARG, "bad B=%d H=%d", B, H);
  if (B == 0) return ok();
  stq_status st = check_ptrs({d_S, d_q, d_k, d_v, d_gate, d_beta, d_out});
  if (st != STQ_OK) return st;
  cudaError_t e = stq::launch_fp32_step(kind, B, H, d_S, d_q, d_k, d_v, d_gate, d_beta, d_out,
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stq_fp32_decode_step launch");
  return ok();
}

stq_status stq_pool_check(stq_pool* pool, void* stream) {
  if (pool == nullptr) return fail(STQ_ERR_INVALID_ARG, "pool is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t bits[4] = {0, 0, 0, 0};
  e = cudaMemcpy(bits, pool->dev.err, sizeof(bits), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read of device error word");
  if (bits[0] != 0) {
    const uint32_t zero[4] = {0, 0, 0, 0};
    e = cudaMemcpy(pool->dev.err, zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear of device error word");
    if (bits[0] & stq::ERR_SLOT_RANGE)
      return fail(STQ_ERR_DEVICE_CHECK, "a slot index was outside [0, n_slots); those heads were skipped");
    if (bits[0] & stq::ERR_CODE)
      return fail(STQ_ERR_DEVICE_CHECK, "a stored code was 0, which the quantiser never writes: "
                                        "a slot was decoded before stq_quantize_init or is corrupted");
    if (bits[0] & stq::ERR_NONFINITE)
      return fail(STQ_ERR_DEVICE_CHECK, "the updated state held a NaN or an infinity (non-finite inputs?)");
    return fail(STQ_ERR_DEVICE_CHECK, "device error bits 0x%x", bits[0]);
  }
  return ok();
}

}  // extern "C"
