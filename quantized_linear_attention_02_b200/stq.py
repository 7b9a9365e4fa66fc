"""Thin Python binding of the C ABI in include/stq.h (argument marshalling only).

Every step of the decode path runs in the CUDA library libstq.so built from csrc/;
torch only provides device memory and streams. Nothing here computes on the host,
and there is no fallback: a missing library raises at load time.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstq.so")

STQ_GDN, STQ_KDA = 0, 1
STATIC_STAGING_BYTES = 8 << 20     # STQ_STATIC_STAGING_BYTES of include/stq.h
D = 128
PIVOT_BITS = 16
KINDS = {"gdn": STQ_GDN, "kda": STQ_KDA}
SCHEMES = {"stepquant": 0, "row_absmax": 1}


class StqError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"stq status {status}: {msg}")
        self.status = status


class _Desc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("n_slots", ctypes.c_int), ("H", ctypes.c_int),
                ("d", ctypes.c_int), ("unit_bits", ctypes.POINTER(ctypes.c_uint8)),
                ("omega", ctypes.POINTER(ctypes.c_float)), ("scheme", ctypes.c_int),
                ("scale_bits", ctypes.c_int)]


class _Sizes(ctypes.Structure):
    _fields_ = [("codes_bytes", ctypes.c_size_t), ("scales_bytes", ctypes.c_size_t),
                ("pivots_bytes", ctypes.c_size_t), ("meta_bytes", ctypes.c_size_t),
                ("slot_code_bytes", ctypes.c_size_t), ("n_pivot_rows", ctypes.c_int),
                ("max_head_bytes", ctypes.c_int)]


_lib = None
_vp = ctypes.c_void_p
_i = ctypes.c_int


def lib():
    """Load libstq.so (built in-tree by build.py; the environment variable STQ_LIBRARY may
    name another build of it, e.g. the checked one); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = os.environ.get("STQ_LIBRARY", LIB_PATH)
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m quantized_linear_attention_02_b200.build`")
    L = ctypes.CDLL(path)
    sig = {
        "stq_pool_layout": (_i, [ctypes.POINTER(_Desc), ctypes.POINTER(_Sizes)]),
        "stq_pool_create": (_i, [ctypes.POINTER(_Desc), _vp, _vp, _vp, _vp, ctypes.POINTER(_vp)]),
        "stq_pool_destroy": (None, [_vp]),
        "stq_quantize_init": (_i, [_vp, _vp, _i, _vp, _vp]),
        "stq_decode_step": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "stq_decode_step_host_staging_bytes": (ctypes.c_size_t, [_vp, _i]),
        "stq_decode_step_host": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                      ctypes.c_size_t, _vp]),
        "stq_decode_step_host_static": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "stq_pipeline_staging_bytes": (ctypes.c_size_t, [_vp, _i]),
        "stq_pipeline_create": (_i, [_vp, _i, _vp, ctypes.c_size_t, ctypes.POINTER(_vp)]),
        "stq_pipeline_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "stq_pipeline_finish": (_i, [_vp, _vp]),
        "stq_pipeline_destroy": (None, [_vp]),
        "stq_dequantize": (_i, [_vp, _vp, _i, _vp, _vp]),
        "stq_fp32_decode_step": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
        "stq_pool_check": (_i, [_vp, _vp]),
        "stq_row_sq_error": (_i, [_vp, _vp, _i, _vp, _i, _vp]),
        "stq_row_error_at_widths": (_i, [_vp, _vp, _i, _vp, _vp, _i, _vp, _vp]),
        "stq_lifetime_weights": (_i, [_vp, _i, _i, _vp]),
        "stq_unit_distortion": (_i, [_i, _i, _i, _vp, _vp, _vp]),
        "stq_allocate_bits": (_i, [_i, _i, _vp, _vp, _vp, ctypes.c_double, _i, _vp]),
        "stq_issue_rate_probe": (_i, [_i, _i, _i, _vp, _vp]),
        "stq_last_error": (ctypes.c_char_p, []),
        "stq_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(status):
    if status != 0:
        raise StqError(status, lib().stq_last_error().decode())


def _desc(kind, n_slots, unit_bits, omega, scheme="stepquant", scale_bits=32):
    ub = np.ascontiguousarray(unit_bits, dtype=np.uint8)
    om = np.ascontiguousarray(omega, dtype=np.float32)
    H = om.shape[0]
    d = _Desc(KINDS[kind] if isinstance(kind, str) else int(kind), int(n_slots), int(H), D,
              ub.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
              om.ctypes.data_as(ctypes.POINTER(ctypes.c_float)),
              SCHEMES[scheme] if isinstance(scheme, str) else int(scheme), int(scale_bits))
    return d, (ub, om)   # keep the arrays alive with the struct


def layout(kind, n_slots, unit_bits, omega, scheme="stepquant", scale_bits=32) -> dict:
    """Buffer sizes of a pool (host only; no CUDA call)."""
    d, keep = _desc(kind, n_slots, unit_bits, omega, scheme, scale_bits)
    s = _Sizes()
    _check(lib().stq_pool_layout(ctypes.byref(d), ctypes.byref(s)))
    return {f: getattr(s, f) for f, _ in _Sizes._fields_}


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, dtype, name, numel=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")
    return ctypes.c_void_p(t.data_ptr())


class Pool:
    """A packed state pool on the current CUDA device. The buffers are torch tensors
    owned here; the library handle only references them."""

    def __init__(self, kind, n_slots, unit_bits, omega, device=None, scheme="stepquant", scale_bits=32):
        import torch
        self.kind = kind
        self.kind_id = KINDS[kind]
        self.scheme = scheme
        self.scale_bits = int(scale_bits)
        self.n_slots = int(n_slots)
        self.unit_bits = np.ascontiguousarray(unit_bits, dtype=np.uint8)
        self.omega = np.ascontiguousarray(omega, dtype=np.float32)
        self.H = self.omega.shape[0]
        self.sizes = layout(kind, n_slots, self.unit_bits, self.omega, scheme, scale_bits)
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        s = self.sizes
        self.codes = torch.zeros(max(s["codes_bytes"], 16), dtype=torch.uint8, device=dev)
        sdt = torch.float16 if self.scale_bits == 16 else torch.float32
        self.scales = torch.zeros(s["scales_bytes"] // (2 if self.scale_bits == 16 else 4), dtype=sdt, device=dev)
        self.pivots = torch.zeros(max(s["pivots_bytes"] // 2, 8), dtype=torch.float16, device=dev)
        self.meta = torch.zeros(s["meta_bytes"], dtype=torch.uint8, device=dev)
        d, keep = _desc(kind, n_slots, self.unit_bits, self.omega, scheme, scale_bits)
        h = ctypes.c_void_p()
        _check(lib().stq_pool_create(ctypes.byref(d), ctypes.c_void_p(self.codes.data_ptr()),
                                     ctypes.c_void_p(self.scales.data_ptr()),
                                     ctypes.c_void_p(self.pivots.data_ptr()),
                                     ctypes.c_void_p(self.meta.data_ptr()), ctypes.byref(h)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib().stq_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # views of the buffers in the pool's layout
    def codes_view(self):
        return self.codes[: self.sizes["codes_bytes"]].view(self.n_slots, -1)

    def scales_view(self):
        return self.scales.view(self.n_slots, self.H, 2, D)

    def pivots_view(self):
        n = self.sizes["n_pivot_rows"]
        return self.pivots[: self.n_slots * n * D].view(self.n_slots, n, D)

    def _slots(self, slots):
        import torch
        return _ptr(slots, torch.int32, "slots")

    def quantize_init(self, slots, S, stream=None):
        import torch
        B = slots.numel()
        _check(lib().stq_quantize_init(self.handle, self._slots(slots), B,
                                       _ptr(S, torch.float32, "S", B * self.H * D * D), _stream(stream)))

    def decode_step(self, slots, q, k, v, gate, beta, out, stream=None):
        import torch
        B = slots.numel()
        n = B * self.H * D
        ng = B * self.H if self.kind_id == STQ_GDN else n
        _check(lib().stq_decode_step(self.handle, self._slots(slots), B,
                                     _ptr(q, torch.float32, "q", n), _ptr(k, torch.float32, "k", n),
                                     _ptr(v, torch.float32, "v", n), _ptr(gate, torch.float32, "gate", ng),
                                     _ptr(beta, torch.float32, "beta", B * self.H),
                                     _ptr(out, torch.float32, "out", n), _stream(stream)))

    def host_staging_bytes(self, B):
        return int(lib().stq_decode_step_host_staging_bytes(self.handle, int(B)))

    def decode_step_host(self, slots, h_q, h_k, h_v, h_gate, h_beta, h_out, staging, stream=None):
        """Decode step with host (pinned) input/output tensors; copies run inside the
        library call on `stream`."""
        import torch
        B = slots.numel()
        for name, t in (("q", h_q), ("k", h_k), ("v", h_v), ("gate", h_gate), ("beta", h_beta), ("out", h_out)):
            if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError(f"host {name} must be a contiguous float32 CPU tensor")
        _check(lib().stq_decode_step_host(
            self.handle, self._slots(slots), B, ctypes.c_void_p(h_q.data_ptr()),
            ctypes.c_void_p(h_k.data_ptr()), ctypes.c_void_p(h_v.data_ptr()),
            ctypes.c_void_p(h_gate.data_ptr()), ctypes.c_void_p(h_beta.data_ptr()),
            ctypes.c_void_p(h_out.data_ptr()), _ptr(staging, torch.uint8, "staging"),
            ctypes.c_size_t(staging.numel()), _stream(stream)))

    def decode_step_host_static(self, slots, h_q, h_k, h_v, h_gate, h_beta, h_out, stream=None):
        """Decode step with host (pinned) tensors and the library's own static device
        staging (no device buffer from the caller; see include/stq.h)."""
        import torch
        B = slots.numel()
        for name, t in (("q", h_q), ("k", h_k), ("v", h_v), ("gate", h_gate), ("beta", h_beta), ("out", h_out)):
            if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError(f"host {name} must be a contiguous float32 CPU tensor")
        _check(lib().stq_decode_step_host_static(
            self.handle, self._slots(slots), B, ctypes.c_void_p(h_q.data_ptr()),
            ctypes.c_void_p(h_k.data_ptr()), ctypes.c_void_p(h_v.data_ptr()),
            ctypes.c_void_p(h_gate.data_ptr()), ctypes.c_void_p(h_beta.data_ptr()),
            ctypes.c_void_p(h_out.data_ptr()), _stream(stream)))

    def row_error_at_widths(self, slots, S, cand_bits, err, stream=None):
        """In-head row errors at candidate widths (stq_row_error_at_widths): S [B, H, 128,
        128] float32 CUDA, err [B, H, 128, len(cand_bits)] float32 CUDA."""
        import torch
        B = slots.numel()
        cb = np.ascontiguousarray(cand_bits, dtype=np.int32)
        _check(lib().stq_row_error_at_widths(
            self.handle, self._slots(slots), B, _ptr(S, torch.float32, "S", B * self.H * D * D),
            cb.ctypes.data_as(ctypes.c_void_p), int(cb.size),
            _ptr(err, torch.float32, "err", B * self.H * D * cb.size), _stream(stream)))

    def pipeline(self, B, staging=None):
        """A Pipeline of host-buffer decode steps of B requests (see Pipeline)."""
        return Pipeline(self, B, staging)

    def dequantize(self, slots, S_out, stream=None):
        import torch
        B = slots.numel()
        _check(lib().stq_dequantize(self.handle, self._slots(slots), B,
                                    _ptr(S_out, torch.float32, "S_out", B * self.H * D * D),
                                    _stream(stream)))

    def check(self, stream=None):
        """Synchronise and raise StqError if a kernel flagged a bad slot index."""
        _check(lib().stq_pool_check(self.handle, _stream(stream)))


def fp32_decode_step(kind, S, q, k, v, gate, beta, out, stream=None):
    """FP32-state decode step in place on S [B, H, 128, 128]."""
    import torch
    B, H = S.shape[0], S.shape[1]
    n = B * H * D
    kid = KINDS[kind]
    ng = B * H if kid == STQ_GDN else n
    _check(lib().stq_fp32_decode_step(kid, B, H, D, _ptr(S, torch.float32, "S", n * D),
                                      _ptr(q, torch.float32, "q", n), _ptr(k, torch.float32, "k", n),
                                      _ptr(v, torch.float32, "v", n), _ptr(gate, torch.float32, "gate", ng),
                                      _ptr(beta, torch.float32, "beta", B * H),
                                      _ptr(out, torch.float32, "out", n), _stream(stream)))


# ---------------------------------------------------------------------------------
# offline calibration (lifetime-aware widths); see include/stq.h
# ---------------------------------------------------------------------------------
def row_sq_error(S, S_hat, err, accumulate=False, stream=None):
    """err[s*128 + i] (+)= sum_j (S - S_hat)^2 over the rows of n_states 128x128 states."""
    import torch
    n = S.numel() // (D * D)
    _check(lib().stq_row_sq_error(_ptr(S, torch.float32, "S", n * D * D),
                                  _ptr(S_hat, torch.float32, "S_hat", n * D * D), n,
                                  _ptr(err, torch.float32, "err", n * D), int(bool(accumulate)),
                                  _stream(stream)))


PROBE_THREADS = 512     # threads per CTA of the issue-rate probe


def issue_rate_probe(mode, blocks, iters, out, stream=None):
    """Launch the issue-rate probe (mode 0: packed FP32 FMA, 1: scalar FP32 FMA, 2: LOP3):
    `blocks` CTAs of 512 threads, 8 chains of `iters` instructions per thread, one float
    per thread into `out`. Returns the lane operations the launch performs."""
    import torch
    _check(lib().stq_issue_rate_probe(int(mode), int(blocks), int(iters),
                                      _ptr(out, torch.float32, "out", blocks * PROBE_THREADS),
                                      _stream(stream)))
    return blocks * PROBE_THREADS * 8 * iters * (2 if mode == 0 else 1)


def _host(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def lifetime_weights(ell, horizon=1024):
    """L_u = sum_{j<horizon} exp(2 j ell_u) (host)."""
    e = _host(ell, np.float64).reshape(-1)
    out = np.empty_like(e)
    _check(lib().stq_lifetime_weights(e.ctypes.data, e.size, int(horizon), out.ctypes.data))
    return out.reshape(np.shape(ell))


def unit_distortion(kind, row_err, omega):
    """Per-unit distortion from row errors [N, H, 128] (host float32)."""
    e = _host(row_err, np.float32)
    N, H = e.shape[0], e.shape[1]
    om = _host(omega, np.float32)
    out = np.empty(H if KINDS[kind] == STQ_GDN else H * D, np.float64)
    _check(lib().stq_unit_distortion(KINDS[kind], N, H, e.ctypes.data, om.ctypes.data, out.ctypes.data))
    return out


def allocate_bits(lifetime, dist, cand_bits, budget, n_pivots):
    """Widths per unit (16 = FP16 pivot) minimising the lifetime-weighted distortion."""
    L = _host(lifetime, np.float64).reshape(-1)
    Dm = _host(dist, np.float64)
    cb = _host(cand_bits, np.int32)
    out = np.empty(L.size, np.uint8)
    _check(lib().stq_allocate_bits(L.size, cb.size, cb.ctypes.data, L.ctypes.data, Dm.ctypes.data,
                                   float(budget), int(n_pivots), out.ctypes.data))
    return out


class Pipeline:
    """stq_pipeline_* of include/stq.h: host-buffer decode steps whose copies overlap the
    previous and next steps inside the library. `step` enqueues one step and returns once
    the previous step's readout is in its host tensor; `finish` waits for the last one.
    The staging buffer (a uint8 CUDA tensor, allocated here if not given) and the pool
    must outlive the pipeline."""

    def __init__(self, pool, B, staging=None):
        import torch
        self.pool, self.B = pool, int(B)
        need = int(lib().stq_pipeline_staging_bytes(pool.handle, self.B))
        if staging is None:
            staging = torch.empty(need, dtype=torch.uint8, device=pool.codes.device)
        self.staging = staging
        h = ctypes.c_void_p()
        _check(lib().stq_pipeline_create(pool.handle, self.B, _ptr(staging, torch.uint8, "staging"),
                                         ctypes.c_size_t(staging.numel()), ctypes.byref(h)))
        self.handle = h

    def step(self, slots, h_q, h_k, h_v, h_gate, h_beta, h_out, stream=None):
        import torch
        if slots.numel() != self.B:
            raise ValueError(f"the pipeline runs {self.B} requests, got {slots.numel()} slots")
        for name, t in (("q", h_q), ("k", h_k), ("v", h_v), ("gate", h_gate), ("beta", h_beta), ("out", h_out)):
            if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError(f"host {name} must be a contiguous float32 CPU tensor")
        _check(lib().stq_pipeline_step(
            self.handle, self.pool._slots(slots), ctypes.c_void_p(h_q.data_ptr()),
            ctypes.c_void_p(h_k.data_ptr()), ctypes.c_void_p(h_v.data_ptr()),
            ctypes.c_void_p(h_gate.data_ptr()), ctypes.c_void_p(h_beta.data_ptr()),
            ctypes.c_void_p(h_out.data_ptr()), _stream(stream)))

    def finish(self, stream=None):
        _check(lib().stq_pipeline_finish(self.handle, _stream(stream)))

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib().stq_pipeline_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # pragma: no cover - interpreter shutdown
            pass
