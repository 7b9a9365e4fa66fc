"""Plain NumPy oracle of the packed Delta-rule state decode step.

Test infrastructure only (see the package docstring). Every array operation here
is a float32 IEEE operation rounded to nearest-even, unless it says float64.

Citations name the page and section of the web pages on "STEPQuant: When and Where
Errors Matter in Delta-Rule Recurrent State Quantization" (arXiv 2609.38169):
  bloombook   = bloombook.cn tutorial (sections numbered one..six)
  lens        = singularity-lens.com summary
  ai-trend    = ai-trend.me review
  zhichai     = zhichai.net forum page

Readings taken where the pages are silent:
  * Arithmetic precision: the state and its update are float32 (the pages compare
    everything against an FP32 state and read out in floating point before
    requantising: lens, decode-order paragraph; zhichai forum reply).
  * The decay D_t is folded into the row scale before dequantising:
    S'_ij = (Q_ij * (d_i * r_i)) * c_j. D_t is diagonal over key rows, so this is the
    same matrix as D_t * (r c Q).
  * Every sum over the 128 entries of a row or a column is a balanced binary tree:
    adjacent pairs first, then adjacent pairs of those, and so on (`tree_sum`). A sum
    of products a_i b_i forms each adjacent pair with one fused multiply-add,
    fma(a_2m, b_2m, a_2m+1 * b_2m+1) (`tree_dot`); the state update is the fused
    S_ij = fma(k_i, delta_j, S'_ij). Every other product is rounded on its own. The
    quantiser's x = y * (1/c) is taken exactly before rounding to an integer.
  * Row scale r_i = mean_j |S_ij| * (omega_i / mean omega)^(-1/2); the column scale
    starts at c_j = max_i |S_ij| / (r_i qmax_i) and takes exactly two omega-weighted
    least-squares steps; the stored codes are requantised with the final c.
  * The least-squares sums use r_i * y_ij (y_ij = S_ij / r_i as rounded) for S_ij:
    num_j = sum_i p_ij y_ij, den_j = sum_i p_ij Q_ij with p_ij = (omega_i r_i^2) Q_ij.
  * Codes are symmetric, Q in [-qmax, qmax], qmax = 2^(b-1) - 1, stored biased as
    u = Q + 2^(b-1). A row of b-bit codes is a little-endian bit stream: code j takes
    bits [b*j, b*j + b).
  * Degenerate cases: a zero row scale gives an all-zero row of Q and no weight; a
    zero column scale gives an all-zero column of Q; a column whose least-squares
    denominator is 0 keeps its previous scale. A scale below 2^-126 (the smallest
    normal float32) is treated as zero when its reciprocal is taken.
  * FP16 pivot rows are stored as the float16 rounding of the updated float32 state
    and take no part in the refit.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
F64 = np.float64
PIVOT_BITS = 16


# ----------------------------------------------------------------------------------
# small helpers
# ----------------------------------------------------------------------------------

def qmax_of(bits):
    """Largest code magnitude of a symmetric b-bit code: 2^(b-1) - 1 (1, 7, 31, 127).
    Pivot rows (16) get 0: they hold no codes."""
    bits = np.asarray(bits, dtype=np.int64)
    return np.where(bits == PIVOT_BITS, 0, (1 << (bits - 1)) - 1)


def bias_of(bits):
    """Offset of the stored unsigned code: u = Q + 2^(b-1)."""
    bits = np.asarray(bits, dtype=np.int64)
    return np.where(bits == PIVOT_BITS, 0, 1 << (bits - 1))


def tree_sum(x, axis):
    """Sum along `axis` (length a power of two) as a balanced binary tree in float32:
    x0+x1, x2+x3, ..., then (x0+x1)+(x2+x3), and so on."""
    x = np.moveaxis(np.asarray(x, dtype=F32), axis, -1)
    n = x.shape[-1]
    assert n & (n - 1) == 0, "tree_sum needs a power-of-two length"
    while x.shape[-1] > 1:
        x = x[..., 0::2] + x[..., 1::2]
    return x[..., 0]


def fma32(a, b, c):
    """float32 fused multiply-add a*b + c with one rounding (nearest-even).

    a*b is exact in float64; a + b in float64 is made "round to odd" (if the float64
    sum is inexact and its last bit is even, step one float64 ulp towards the exact
    value, found with the error-free two-sum), so that the final rounding to float32
    equals the rounding of the exact value (round-to-odd with 53 >= 24 + 2 bits;
    Boldo and Melquiond, "Emulation of FMA and correctly rounded sums: proved
    algorithms using rounding to odd", IEEE TC 2008)."""
    a = np.asarray(a, dtype=F32).astype(F64)
    b = np.asarray(b, dtype=F32).astype(F64)
    c = np.asarray(c, dtype=F32).astype(F64)
    p = a * b
    s = np.asarray(p + c)
    bp = s - p
    err = (p - (s - bp)) + (c - bp)
    bits = s.view(np.int64)
    fix = (err != 0) & ((bits & 1) == 0)
    # one float64 ulp towards the exact value: +1 on the bit pattern when s and err
    # have the same sign (away from zero), -1 otherwise (s == 0 implies err == 0)
    step = np.where((s > 0) == (err > 0), 1, -1)
    bits = bits + np.where(fix, step, 0)
    return bits.view(F64).astype(F32)


def tree_dot(a, b, axis):
    """sum_i a_i b_i along `axis` (power-of-two length): adjacent products paired by
    one fused multiply-add, fma(a_2m, b_2m, a_2m+1 * b_2m+1), then `tree_sum`."""
    a = np.moveaxis(np.asarray(a, dtype=F32), axis, -1)
    b = np.moveaxis(np.asarray(b, dtype=F32), axis, -1)
    a, b = np.broadcast_arrays(a, b)
    pairs = fma32(a[..., 0::2], b[..., 0::2], a[..., 1::2] * b[..., 1::2])
    return tree_sum(pairs, axis=-1)


def row_gain(omega):
    """g_i = (omega_i / mean_i omega)^(-1/2) for each head, evaluated in float64
    (mean = sequential float64 sum / d, then divide, square root, reciprocal) and
    rounded once to float32. The row scale folds in the row influence so that
    high-influence rows get finer steps (lens, dual-axis paragraph; bloombook
    section 4 gives r_i with a w_i^(-1/2) factor)."""
    w = np.asarray(omega, dtype=F64)
    d = w.shape[-1]
    mean = np.cumsum(w, axis=-1)[..., -1:] / d
    return (1.0 / np.sqrt(w / mean)).astype(F32)


# ----------------------------------------------------------------------------------
# code packing (one row = one little-endian bit stream)
# ----------------------------------------------------------------------------------

def pack_row(u, bits):
    """Pack unsigned codes u[..., d] (each < 2^bits) into bytes[..., d*bits/8]:
    bit t of code j goes to bit b*j + t of the stream, and stream bit n goes to bit
    n % 8 of byte n // 8. For b = 6 this packs four codes into three bytes."""
    u = np.asarray(u, dtype=np.int64)
    d = u.shape[-1]
    assert (d * bits) % 8 == 0
    assert np.all((u >= 0) & (u < (1 << bits)))
    stream = (u[..., :, None] >> np.arange(bits)) & 1            # [..., d, bits]
    stream = stream.reshape(u.shape[:-1] + (d * bits // 8, 8))   # [..., nbytes, 8]
    return (stream << np.arange(8)).sum(axis=-1).astype(np.uint8)


def unpack_row(buf, bits, d):
    """Inverse of pack_row: bytes[..., d*bits/8] -> codes[..., d] (int64)."""
    buf = np.asarray(buf, dtype=np.int64)
    stream = (buf[..., :, None] >> np.arange(8)) & 1             # [..., nbytes, 8]
    stream = stream.reshape(buf.shape[:-1] + (d, bits))
    return (stream << np.arange(bits)).sum(axis=-1)


# ----------------------------------------------------------------------------------
# pool layout: where each head's bytes live inside one slot
# ----------------------------------------------------------------------------------

class Layout:
    """Byte layout of one state slot, from the per-row widths [H, d].

    codes : rows of non-pivot units, head after head, row after row; row i of head h
            takes d*b/8 bytes.
    pivots: float16 rows (d*2 bytes each) of the pivot rows, in (head, row) order.
    scales: float32 r[d] then c[d] for every head (pivot heads included).
    """

    def __init__(self, row_bits):
        self.row_bits = np.asarray(row_bits, dtype=np.int64)
        H, d = self.row_bits.shape
        self.H, self.d = H, d
        code_len = np.where(self.row_bits == PIVOT_BITS, 0, d * self.row_bits // 8)
        self.row_code_offset = np.zeros((H, d), dtype=np.int64)
        off = 0
        for h in range(H):
            for i in range(d):
                self.row_code_offset[h, i] = off
                off += int(code_len[h, i])
        self.code_len = code_len
        self.slot_code_bytes = off
        self.pivot_index = -np.ones((H, d), dtype=np.int64)
        p = 0
        for h in range(H):
            for i in range(d):
                if self.row_bits[h, i] == PIVOT_BITS:
                    self.pivot_index[h, i] = p
                    p += 1
        self.n_pivot_rows = p
        self.slot_scale_floats = H * 2 * d


class Pool:
    """Host image of a state pool: codes [n_slots, slot_code_bytes] uint8,
    scales [n_slots, H, 2, d] float32, pivots [n_slots, n_pivot_rows, d] float16."""

    def __init__(self, layout: Layout, n_slots: int, scale16: bool = False):
        self.layout = layout
        self.n_slots = n_slots
        self.codes = np.zeros((n_slots, layout.slot_code_bytes), dtype=np.uint8)
        # compact pools keep r and c as float16 (values already float16-representable)
        self.scales = np.zeros((n_slots, layout.H, 2, layout.d), dtype=np.float16 if scale16 else F32)
        self.pivots = np.zeros((n_slots, max(layout.n_pivot_rows, 0), layout.d), dtype=np.float16)

    def write_heads(self, slots, u, r, c, piv):
        """Store codes u[B,H,d,d] (biased), scales r,c [B,H,d], pivot rows piv[B,H,d,d]
        (float16, only pivot rows read) for the given slots."""
        L = self.layout
        for bi, s in enumerate(slots):
            for h in range(L.H):
                for i in range(L.d):
                    b = int(L.row_bits[h, i])
                    if b == PIVOT_BITS:
                        self.pivots[s, L.pivot_index[h, i]] = piv[bi, h, i]
                    else:
                        o = L.row_code_offset[h, i]
                        self.codes[s, o:o + L.code_len[h, i]] = pack_row(u[bi, h, i], b)
                self.scales[s, h, 0] = r[bi, h]
                self.scales[s, h, 1] = c[bi, h]

    def read_heads(self, slots):
        """Return (u[B,H,d,d] int64, r, c [B,H,d] float32, piv [B,H,d,d] float16)."""
        L = self.layout
        B = len(slots)
        u = np.zeros((B, L.H, L.d, L.d), dtype=np.int64)
        piv = np.zeros((B, L.H, L.d, L.d), dtype=np.float16)
        for bi, s in enumerate(slots):
            for h in range(L.H):
                for i in range(L.d):
                    b = int(L.row_bits[h, i])
                    if b == PIVOT_BITS:
                        piv[bi, h, i] = self.pivots[s, L.pivot_index[h, i]]
                    else:
                        o = L.row_code_offset[h, i]
                        u[bi, h, i] = unpack_row(self.codes[s, o:o + L.code_len[h, i]], b, L.d)
        r = self.scales[list(slots), :, 0].astype(F32)
        c = self.scales[list(slots), :, 1].astype(F32)
        return u, r, c, piv


# ----------------------------------------------------------------------------------
# the method
# ----------------------------------------------------------------------------------

def dequantize(u, r, c, piv, row_bits, decay=None):
    """Restore the float32 state from codes (bloombook section 4: X_ij = r_i c_j z_ij;
    lens decode-order paragraph: the previous state is restored first).

    u[..., d, d] biased codes, r/c [..., d], piv [..., d, d] float16, row_bits [H, d]
    broadcast over the leading batch axis. decay[..., d] (per key row, the diagonal of
    D_t) is folded into the row scale: S'_ij = (Q_ij * (d_i r_i)) * c_j; pivot rows
    give S'_ij = d_i * h_ij. decay=None means no decay (plain export)."""
    row_bits = np.asarray(row_bits)
    pivot = row_bits == PIVOT_BITS
    Q = (np.asarray(u, dtype=np.int64) - bias_of(row_bits)[..., None]).astype(F32)
    r = np.asarray(r, dtype=F32)
    if decay is not None:
        rd = np.asarray(decay, dtype=F32) * r
    else:
        rd = r
    S = (Q * rd[..., :, None]) * np.asarray(c, dtype=F32)[..., None, :]
    P = np.asarray(piv).astype(F32)
    if decay is not None:
        P = np.asarray(decay, dtype=F32)[..., :, None] * P
    return np.where(pivot[..., None], P, S).astype(F32)


def delta_update(Sp, k, v, beta):
    """Gated delta rule on an already-decayed state S' = D_t S_{t-1}
    (bloombook section 2: S_t = (I - beta k k^T) D_t S_{t-1} + beta k v^T):
        u_j = sum_i k_i S'_ij,  delta_j = beta (v_j - u_j),  S_ij = S'_ij + k_i delta_j,
    which is the same matrix as the printed form. Sp [..., d, d], k/v [..., d],
    beta [...]."""
    Sp = np.asarray(Sp, dtype=F32)
    k = np.asarray(k, dtype=F32)
    u = tree_dot(k[..., :, None], Sp, axis=-2)
    delta = np.asarray(beta, dtype=F32)[..., None] * (np.asarray(v, dtype=F32) - u)
    return fma32(k[..., :, None], delta[..., None, :], Sp)


def readout(S, q):
    """o_j = sum_i q_i S_ij from the float32 state (bloombook section 3: the output
    is the state times the query), evaluated in float64 and rounded to float32."""
    S64 = np.asarray(S, dtype=F64)
    q64 = np.asarray(q, dtype=F64)
    return np.einsum("...ij,...i->...j", S64, q64).astype(F32)


def _quantise(y, inv_c, qm):
    """Q_ij = clamp(rint(y_ij * inv_c_j), -qmax_i, qmax_i); the product of two float32
    numbers is exact in float64, so rint sees the exact product."""
    x = np.asarray(y, dtype=F64) * np.asarray(inv_c, dtype=F64)[..., None, :]
    return np.clip(np.rint(x), -qm[..., :, None], qm[..., :, None]).astype(F32)


TINY = F32(np.finfo(np.float32).tiny)   # 2^-126, the smallest normal float32


def _recip(a):
    """float32 1/a for a scale a >= 2^-126; a smaller scale counts as zero and gets 0
    (its reciprocal would overflow)."""
    a = np.asarray(a, dtype=F32)
    ok = a >= TINY
    safe = np.where(ok, a, F32(1))
    return np.where(ok, F32(1) / safe, F32(0)).astype(F32)


def _half(x):
    """Round float32 values to IEEE binary16 (to nearest, ties to even) and back."""
    return np.asarray(x, dtype=F32).astype(np.float16).astype(F32)


def refit(S, omega, row_bits, n_ls=2, scale16=False):
    """Dual-axis refit of a float32 state and its codes (bloombook section 4,
    X_ij = r_i c_j z_ij with an omega-weighted column fit; lens dual-axis paragraph;
    ai-trend Method (2)).

    S [..., d, d] float32; omega [H, d] float32 (> 0); row_bits [H, d].
    scale16: compact storage of the scales as binary16 (reading: r is rounded to
    binary16 as soon as it is formed, so y, the weights and the codes use the stored r;
    the column start and both least-squares steps run in float32; the final c is
    rounded to binary16 before the codes are requantised with it, so the stored
    (r, c, Q) stay consistent).

    Returns (u biased codes int64 [..., d, d], r [..., d], c [..., d],
    piv float16 [..., d, d] (meaningful on pivot rows only))."""
    S = np.asarray(S, dtype=F32)
    row_bits = np.asarray(row_bits)
    pivot = row_bits == PIVOT_BITS
    d = S.shape[-1]
    qm = qmax_of(row_bits).astype(F32)
    inv_qm = _recip(qm)
    g = row_gain(omega)
    # row scale: mean |S_ij| over the row times g_i (division by d is exact)
    m = tree_sum(np.abs(S), axis=-1) * F32(1.0 / d)
    r = np.where(pivot, F32(0), m * g).astype(F32)
    if scale16:
        r = _half(r)
    inv_r = _recip(r)
    y = S * inv_r[..., :, None]
    # column scale start: no element clips
    c = np.max(np.abs(y) * inv_qm[..., :, None], axis=-2).astype(F32)
    b = (np.asarray(omega, dtype=F32) * (r * r)).astype(F32)
    for _ in range(n_ls):
        Q = _quantise(y, _recip(c), qm)
        p = b[..., :, None] * Q
        num = tree_dot(p, y, axis=-2)
        den = tree_dot(p, Q, axis=-2)
        safe = np.where(den > 0, den, F32(1))
        c = np.where(den > 0, num / safe, c).astype(F32)
    if scale16:
        c = _half(c)
    Q = _quantise(y, _recip(c), qm)
    u = (Q.astype(np.int64) + bias_of(row_bits)[..., None])
    u = np.where(pivot[..., None], 0, u)
    piv = np.where(pivot[..., None], S, F32(0)).astype(np.float16)
    return u, r, c, piv


def absmax_quantise(S, row_bits, scale16=False):
    """The uniform baseline quantiser of the pages: symmetric per-key-row absmax INT-b
    (lens, calibration and evaluation-setup paragraphs name symmetric INT4/6/8 per-row
    absmax quantisers as the uniform comparison). Reading: the row scale is
    r_i = max_j |S_ij| * (1/qmax_i) with 1/qmax_i rounded once (the same form as the
    dual-axis column start), codes Q_ij = clamp(rint(S_ij * (1/r_i)), -qmax_i, qmax_i)
    with the product taken exactly, and the column scales are all 1, so the stored pool
    has the dual-axis layout and dequantises as (Q r) * 1. Pivot rows: float16 as in
    `refit`; a head whose rows are all pivots stores r = c = 0 as under `refit`.

    Returns (u, r, c, piv) like `refit`."""
    S = np.asarray(S, dtype=F32)
    row_bits = np.asarray(row_bits)
    pivot = row_bits == PIVOT_BITS
    qm = qmax_of(row_bits).astype(F32)
    inv_qm = _recip(qm)
    m = np.max(np.abs(S), axis=-1)
    r = np.where(pivot, F32(0), m * inv_qm).astype(F32)
    if scale16:        # compact scales: the codes are fitted to the stored binary16 r
        r = _half(r)
    x = S.astype(F64) * _recip(r).astype(F64)[..., :, None]   # exact product
    Q = np.clip(np.rint(x), -qm[..., :, None], qm[..., :, None]).astype(F32)
    u = (Q.astype(np.int64) + bias_of(row_bits)[..., None])
    u = np.where(pivot[..., None], 0, u)
    # unit column scales; a head without any quantised row stores c = 0, like its r
    has_codes = np.any(~pivot, axis=-1)
    c = np.broadcast_to(np.where(has_codes, F32(1), F32(0))[..., None],
                        S.shape[:-2] + (S.shape[-1],)).astype(F32)
    piv = np.where(pivot[..., None], S, F32(0)).astype(np.float16)
    return u, r, c, piv


def fp32_step(S_prev, q, k, v, decay, beta):
    """One FP32-state decode step (the unquantised path the pages compare against):
    S' = D_t S_{t-1} row-wise, the gated delta update, then the readout."""
    Sp = (np.asarray(decay, dtype=F32)[..., :, None] * np.asarray(S_prev, dtype=F32)).astype(F32)
    S = delta_update(Sp, k, v, beta)
    return S, readout(S, q)


def decode_step(u, r, c, piv, row_bits, omega, q, k, v, decay, beta, n_ls=2, scheme="stepquant",
                scale16=False):
    """One packed-state decode step in the order the pages give (lens decode-order
    paragraph; bloombook section 4, fused kernel paragraph): restore the previous
    state, apply the gated delta update in floating point, read the output from the
    updated float32 state, then refit and requantise for storage.

    decay is per key row [..., d] (GDN: the head's alpha repeated over rows).
    scheme "stepquant" requantises with `refit`, "row_absmax" with `absmax_quantise`;
    scale16 stores the scales as binary16.
    Returns (u, r, c, piv, o, S_float32_before_requantisation)."""
    Sp = dequantize(u, r, c, piv, row_bits, decay=decay)
    S = delta_update(Sp, k, v, beta)
    o = readout(S, q)
    if scheme == "row_absmax":
        u2, r2, c2, piv2 = absmax_quantise(S, row_bits, scale16=scale16)
    else:
        u2, r2, c2, piv2 = refit(S, omega, row_bits, n_ls=n_ls, scale16=scale16)
    return u2, r2, c2, piv2, o, S


def gate_rows(gate, kind, d):
    """Per-row decay from the gate input: GDN [..] -> repeated over d rows; KDA as is."""
    gate = np.asarray(gate, dtype=F32)
    if kind == "gdn":
        return np.repeat(gate[..., None], d, axis=-1)
    return gate


def fp32_warmup(w_steps_inputs, kind, d, S0):
    """Run FP32 steps from S0 over a list of StepInputs-like objects (q,k,v,gate,beta
    with leading [B, H]); returns the final state."""
    S = np.asarray(S0, dtype=F32)
    for x in w_steps_inputs:
        S, _ = fp32_step(S, x.q, x.k, x.v, gate_rows(x.gate, kind, d), x.beta)
    return S
