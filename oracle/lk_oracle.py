"""Plain CPU oracle for the per-head latent-KV decode path.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
test suite, the package smoke check and the CPU-baseline leg of ``bench.py``
may.  It shares no code, table or constant with the CUDA sources.

Everything here is written for a reader checking it against the two source
pages by eye:

* "WSVD: Weighted Low-Rank Approximation for Fast and Efficient Execution of
  Low-Precision Vision-Language Models" (gist.science summary, ICLR 2026),
  technical summary §2A (per-head SVD: each head's E x H slice of the K/V
  projection is factored to rank r, W^h ~ A^h B^h, and only the per-head latent
  x A^h is stored), §2C (W8A8 / W8A4 quantisation and the fused kernel that
  rebuilds K_h on chip and runs flash-decoding QK^T, softmax, PV on it).
* "LASER: Loss-Aware Singular-value Decomposition and Rank Allocation for
  Efficient Low-Precision Vision-Language Models" (gist.science summary),
  technical summary §2 (non-uniform per-layer/per-head ranks), §3 (hybrid FFN:
  selected channels go through SVD factors, the rest stay dense; RTN
  quantisation of both branches), §4 (fused kernels: projection, latent
  activation, SwiGLU, quant/dequant).

Floating point is float64 unless a step is a quantisation decision, which is
taken in float32 (the kernels' precision) exactly as written below.

Readings taken where the pages are silent (each one is also listed in the
design notes):

* Quantiser: symmetric absmax, no zero point, round-half-to-even ("RTN" on the
  LASER page §3), codes clamped to [-127, 127] (int8) or [-7, 7] (int4).
  The scale is the correctly-rounded float32 quotient absmax/127 (int8) or
  fp16(fl32(absmax/7)) saturated to the largest finite fp16 (int4).  A zero
  scale (all-zero input, or underflow) gives all-zero codes.  Codes are
  rint(fl32(v / s)), a true division, not a multiply by 1/s.
* int4 groups: g consecutive latent dims share one fp16 scale; the last group
  of a row may be shorter when g does not divide r.  Packing: low nibble holds
  the even dim, high nibble the odd dim, both two's complement.
* No positional encoding (neither page mentions one), so the absorbed form
  (q B_K^T) C^T equals the materialised one.  The rotary extension below
  (attention_rope) is a separate path with its own readings.
* Attention over positions [0, len) where len already counts the token
  appended in the same step.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "quantize_i8", "quantize_i4", "pack_i4", "unpack_i4",
    "dequantize_i8", "dequantize_i4",
    "latent_project_float", "latent_project_w8a8", "quantize_latents",
    "attention_materialized", "attention_absorbed", "latent_attention",
    "linear_w8a8_hybrid", "quantize_rows_i8", "rmsnorm", "swiglu",
    "per_head_svd", "round_bf16", "LatentCache", "decoder_layer_w8a8",
    "hadamard", "latent_rotation", "rotate_latents", "rmsnorm_hadamard",
    "rope_angles", "rope", "attention_rope", "latent_attention_rope",
    "linear_w8a8_outsplit", "ffn_gate_up_swiglu",
]

FP16_MAX = 65504.0


# ---------------------------------------------------------------------------
# Quantisers (WSVD page §2C "W8A8, W8A4"; LASER page §3 "RTN")
# ---------------------------------------------------------------------------

def _fl32_div(a, b):
    """Correctly rounded float32 quotient of float32 operands.

    The quotient is formed in float64 and rounded once to float32; for
    division, float64 (53 bits) carries more than 2*24+2 bits, so the double
    rounding is innocuous and the result equals IEEE single-precision division.
    """
    return (np.asarray(a, np.float32).astype(np.float64)
            / np.asarray(b, np.float32).astype(np.float64)).astype(np.float32)


def quantize_i8(v):
    """int8 absmax quantiser over the last axis.

    v: float32 [..., r].  Returns (codes int8 [..., r], scale float32 [...]).
    scale = fl32(max|v| / 127); codes = clamp(rint(fl32(v / scale)), -127, 127);
    a zero scale gives zero codes.
    """
    v = np.asarray(v, dtype=np.float32)
    absmax = np.max(np.abs(v), axis=-1)
    scale = _fl32_div(absmax, np.float32(127.0))
    zero = scale == 0
    safe = np.where(zero, np.float32(1.0), scale)
    ratio = _fl32_div(v, safe[..., None])
    codes = np.clip(np.rint(ratio), -127, 127)
    codes = np.where(zero[..., None], 0, codes)
    return codes.astype(np.int8), scale.astype(np.float32)


def quantize_rows_i8(x):
    """Per-token (per-row) absmax int8 activation quantiser; same rule as quantize_i8."""
    return quantize_i8(x)


def quantize_i4(v, group):
    """int4 grouped absmax quantiser over the last axis.

    v: float32 [..., r]; group g: consecutive dims sharing one fp16 scale
    (n_groups = ceil(r / g)).  Returns (codes int8 [..., r] with values in
    [-7, 7] (unpacked), scales float16 [..., n_groups]).
    scale16 = min(fp16_rn(fl32(absmax_group / 7)), 65504); s = float(scale16);
    codes = clamp(rint(fl32(v / s)), -7, 7); s == 0 gives zero codes.
    """
    v = np.asarray(v, dtype=np.float32)
    r = v.shape[-1]
    n_groups = -(-r // group)
    codes = np.zeros(v.shape, dtype=np.int8)
    scales = np.zeros(v.shape[:-1] + (n_groups,), dtype=np.float16)
    for gi in range(n_groups):
        lo, hi = gi * group, min(r, (gi + 1) * group)
        vg = v[..., lo:hi]
        absmax = np.max(np.abs(vg), axis=-1)
        s32 = _fl32_div(absmax, np.float32(7.0))
        with np.errstate(over="ignore"):
            s16 = s32.astype(np.float16)
        s16 = np.minimum(s16, np.float16(FP16_MAX))
        s = s16.astype(np.float32)
        zero = s == 0
        safe = np.where(zero, np.float32(1.0), s)
        ratio = _fl32_div(vg, safe[..., None])
        c = np.clip(np.rint(ratio), -7, 7)
        c = np.where(zero[..., None], 0, c)
        codes[..., lo:hi] = c.astype(np.int8)
        scales[..., gi] = s16
    return codes, scales


def pack_i4(codes):
    """Pack int4 codes [..., r] (r even) two per byte: low nibble = even dim."""
    c = np.asarray(codes, dtype=np.int8).astype(np.int16)
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_i4(packed, r):
    """Inverse of pack_i4: bytes [..., r/2] -> int8 codes [..., r] in [-8, 7]."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    out = np.empty(p.shape[:-1] + (r,), dtype=np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    out = np.where(out >= 8, out - 16, out)
    return out.astype(np.int8)


def dequantize_i8(codes, scale):
    """c_hat = c * s, float64.  codes [..., r], scale [...]."""
    return np.asarray(codes, np.float64) * np.asarray(scale, np.float64)[..., None]


def dequantize_i4(codes, scales, group):
    """c_hat = c * s_group, float64.  codes [..., r] unpacked, scales [..., n_groups]."""
    c = np.asarray(codes, np.float64)
    s = np.asarray(scales, np.float32).astype(np.float64)
    r = c.shape[-1]
    idx = np.arange(r) // group
    return c * s[..., idx]


# ---------------------------------------------------------------------------
# Latent projection (WSVD page §2A: the per-head latent x A^h is what is cached)
# ---------------------------------------------------------------------------

def latent_project_float(x, A):
    """v = x A in float64 on exact stored values, rounded once to float32.

    x: [M, E] (any float dtype; converted exactly), A: [E, N].
    """
    v = np.asarray(x, np.float64) @ np.asarray(A, np.float64)
    return v.astype(np.float32)


def latent_project_w8a8(x_q, x_scale, A_q, a_scale):
    """W8A8 latent projection.

    acc = x_q A_q exactly (int64); v = fl32(fl32(fl32(acc) * s_x[m]) * s_A[n]),
    each product rounded to float32 in that order (a float32 x float32 product
    is exact in float64, so one rounding to float32 is the IEEE product).
    """
    acc = np.asarray(x_q, np.int64) @ np.asarray(A_q, np.int64)
    v = acc.astype(np.float32)
    v = (v.astype(np.float64) * np.asarray(x_scale, np.float32)[:, None]).astype(np.float32)
    v = (v.astype(np.float64)
         * np.asarray(a_scale, np.float16).astype(np.float32)[None, :]).astype(np.float32)
    return v


def quantize_latents(v, ranks, kind, group):
    """Split v [..., sum(ranks)] into heads and quantise each head's row.

    Returns a list over heads of (codes [..., r_h], scales) with scales float32
    [...] (int8) or float16 [..., n_groups] (int4).
    """
    out = []
    off = 0
    for r in ranks:
        vh = v[..., off:off + r]
        off += r
        if kind == "i8":
            out.append(quantize_i8(vh))
        else:
            out.append(quantize_i4(vh, min(group, r)))
    assert off == v.shape[-1]
    return out


# ---------------------------------------------------------------------------
# Attention (WSVD page §2C fused kernel; K = dequant(C_K) B_K, V = dequant(C_V) B_V)
# ---------------------------------------------------------------------------

def attention_materialized(q, Ck_hat, Cv_hat, B_K, B_V, softmax_scale):
    """softmax(q K^T * scale) V for one (batch, head), with K and V materialised.

    q: [H]; Ck_hat: [T, r_K] dequantised latents; B_K: [r_K, H];
    Cv_hat: [T, r_V]; B_V: [r_V, H].  Returns o: [H] float64.
    """
    K = np.asarray(Ck_hat, np.float64) @ np.asarray(B_K, np.float64)   # [T, H]
    V = np.asarray(Cv_hat, np.float64) @ np.asarray(B_V, np.float64)   # [T, H]
    s = (K @ np.asarray(q, np.float64)) * float(softmax_scale)          # [T]
    s = s - np.max(s)
    p = np.exp(s)
    p = p / np.sum(p)
    return p @ V


def attention_absorbed(q, Ck_hat, Cv_hat, B_K, B_V, softmax_scale):
    """The same attention with q absorbed into latent space (no K or V formed).

    q_t = B_K q (r_K values); s = Ck_hat q_t * scale; u = p^T Cv_hat; o = u B_V.
    Equal to attention_materialized when there is no positional rotation.
    """
    q_t = np.asarray(B_K, np.float64) @ np.asarray(q, np.float64)       # [r_K]
    s = (np.asarray(Ck_hat, np.float64) @ q_t) * float(softmax_scale)
    s = s - np.max(s)
    p = np.exp(s)
    p = p / np.sum(p)
    u = p @ np.asarray(Cv_hat, np.float64)                               # [r_V]
    return u @ np.asarray(B_V, np.float64)


class LatentCache:
    """Logical latent cache for one layer and one of K or V.

    codes[b][h]: int8 [T_b, r_h] (unpacked codes); scales[b][h]: float32 [T_b]
    (int8) or float16 [T_b, n_groups] (int4).
    """

    def __init__(self, batch, ranks, kind, group):
        self.batch = batch
        self.ranks = list(ranks)
        self.kind = kind
        self.group = group
        self.codes = [[np.zeros((0, r), np.int8) for r in ranks] for _ in range(batch)]
        if kind == "i8":
            self.scales = [[np.zeros((0,), np.float32) for _ in ranks] for _ in range(batch)]
        else:
            self.scales = [[np.zeros((0, -(-r // min(group, r))), np.float16) for r in ranks]
                           for _ in range(batch)]

    def length(self, b):
        return self.codes[b][0].shape[0] if self.ranks else 0

    def append(self, b, per_head):
        """per_head: list over heads of (codes [n, r_h], scales) for batch row b."""
        for h, (c, s) in enumerate(per_head):
            self.codes[b][h] = np.concatenate([self.codes[b][h], c], axis=0)
            self.scales[b][h] = np.concatenate([self.scales[b][h], s], axis=0)

    def dequant(self, b, h):
        if self.kind == "i8":
            return dequantize_i8(self.codes[b][h], self.scales[b][h])
        return dequantize_i4(self.codes[b][h], self.scales[b][h], min(self.group, self.ranks[h]))


def latent_attention(q, cache_k, cache_v, B_K_heads, B_V_heads, softmax_scale, materialize=True):
    """Attention for every (b, h) over the whole cache.

    q: [B, n_h, H]; B_K_heads[h]: [r_K_h, H]; B_V_heads[h]: [r_V_h, H].
    Returns o: [B, n_h, H] float64.
    """
    q = np.asarray(q, np.float64)
    Bsz, n_h, H = q.shape
    out = np.zeros((Bsz, n_h, H), np.float64)
    fn = attention_materialized if materialize else attention_absorbed
    for b in range(Bsz):
        for h in range(n_h):
            out[b, h] = fn(q[b, h], cache_k.dequant(b, h), cache_v.dequant(b, h),
                           B_K_heads[h], B_V_heads[h], softmax_scale)
    return out


# ---------------------------------------------------------------------------
# LASER hybrid dense + low-rank linear (LASER page §3), W8A8
# ---------------------------------------------------------------------------

def _requant_latent(acc_U, sx, s_U):
    """The low-rank latent t = fl32(fl32(fl32(acc_U) * s_x) * s_U), requantised
    per token with the int8 absmax rule: returns (t_q, s_t)."""
    t = np.asarray(acc_U).astype(np.float32)
    t = (t.astype(np.float64) * sx[:, None]).astype(np.float32)
    t = (t.astype(np.float64)
         * np.asarray(s_U, np.float16).astype(np.float32)[None, :]).astype(np.float32)
    return quantize_rows_i8(t)


def linear_w8a8_hybrid(x_q, x_scale, dense_idx, lr_idx, W_D, s_D, U, s_U, V, s_V,
                       residual=None):
    """y = x_q[:, D] W_D (dense branch) + requant(x_q[:, not D] U) V (low-rank branch).

    x_q int8 [M, K_in] with per-token float32 scale s_x [M]; dense_idx (D) and
    lr_idx (not D) are disjoint sorted channel lists covering [0, K_in);
    W_D int8 [|D|, N] with fp16 per-output scale s_D [N]; U int8 [|not D|, R]
    with fp16 per-column scale s_U [R]; V int8 [R, N] with fp16 scale s_V [N].

    Low-rank latent: t = fl32(fl32(fl32(acc_U) * s_x) * s_U), requantised per
    token with the int8 absmax rule -> (t_q, s_t).  Output (float64):
    y = acc_D * s_x * s_D + acc_V * s_t * s_V (+ residual).
    Returns (y [M, N] float64, t_q, s_t).
    """
    x = np.asarray(x_q, np.int64)
    sx = np.asarray(x_scale, np.float32)
    M = x.shape[0]
    N = np.asarray(s_D if len(dense_idx) else s_V).shape[0]
    y = np.zeros((M, N), np.float64)
    if len(dense_idx):
        acc_D = x[:, np.asarray(dense_idx)] @ np.asarray(W_D, np.int64)
        y += (acc_D.astype(np.float64) * sx.astype(np.float64)[:, None]
              * np.asarray(s_D, np.float16).astype(np.float64)[None, :])
    t_q = np.zeros((M, 0), np.int8)
    s_t = np.zeros((M,), np.float32)
    if len(lr_idx):
        acc_U = x[:, np.asarray(lr_idx)] @ np.asarray(U, np.int64)
        t_q, s_t = _requant_latent(acc_U, sx, s_U)
        acc_V = t_q.astype(np.int64) @ np.asarray(V, np.int64)
        y += (acc_V.astype(np.float64) * s_t.astype(np.float64)[:, None]
              * np.asarray(s_V, np.float16).astype(np.float64)[None, :])
    if residual is not None:
        y += np.asarray(residual, np.float64)
    return y, t_q, s_t


def linear_w8a8_outsplit(x_q, x_scale, dense_out, lr_out, W_D, s_D, U, s_U, V, s_V):
    """The hybrid linear split on OUTPUT channels (LASER page §3 read as: the
    selected hidden channels of a projection keep dense weights, the rest come
    from the SVD factors).

    x_q int8 [M, K] with per-token float32 scale s_x [M]; dense_out and
    lr_out are disjoint sorted output-channel lists covering [0, N);
    W_D int8 [K, |dense_out|] with fp16 scale s_D [|dense_out|]; U int8 [K, R]
    with fp16 scale s_U [R]; V int8 [R, |lr_out|] with fp16 scale s_V
    [|lr_out|].  Same rules as linear_w8a8_hybrid: the latent
    t = fl32(fl32(fl32(x_q U) * s_x) * s_U) is requantised per token (t_q, s_t);
    y[:, dense_out] = acc_D * s_x * s_D, y[:, lr_out] = acc_V * s_t * s_V
    (float64).  Returns (y [M, N] float64, t_q, s_t).
    """
    x = np.asarray(x_q, np.int64)
    sx = np.asarray(x_scale, np.float32)
    M = x.shape[0]
    N = len(dense_out) + len(lr_out)
    y = np.zeros((M, N), np.float64)
    if len(dense_out):
        acc_D = x @ np.asarray(W_D, np.int64)
        s_dense = np.asarray(s_D, np.float16).astype(np.float64)
        y[:, np.asarray(dense_out)] = acc_D.astype(np.float64) * sx.astype(np.float64)[:, None] * s_dense[None, :]
    t_q = np.zeros((M, 0), np.int8)
    s_t = np.zeros((M,), np.float32)
    if len(lr_out):
        acc_U = x @ np.asarray(U, np.int64)
        t_q, s_t = _requant_latent(acc_U, sx, s_U)
        acc_V = t_q.astype(np.int64) @ np.asarray(V, np.int64)
        s_lr = np.asarray(s_V, np.float16).astype(np.float64)
        y[:, np.asarray(lr_out)] = (acc_V.astype(np.float64) * s_t.astype(np.float64)[:, None]
                                    * s_lr[None, :])
    return y, t_q, s_t


def ffn_gate_up_swiglu(x_q, x_scale, gate, up):
    """silu(gate(x)) * up(x) with both projections split on output channels
    (linear_w8a8_outsplit; gate and up are dicts of its weight arguments).
    Reading: gate and up keep the same hidden channels dense, so channel j of
    both comes from the same kind of branch.  Returns [M, N] float64."""
    g, _, _ = linear_w8a8_outsplit(x_q, x_scale, **gate)
    u, _, _ = linear_w8a8_outsplit(x_q, x_scale, **up)
    return swiglu(g, u)


def swiglu(gate, up):
    """SiLU-gated unit (LASER page §4 fuses it): silu(g) * u = g / (1 + e^-g) * u."""
    g = np.asarray(gate, np.float64)
    u = np.asarray(up, np.float64)
    return g / (1.0 + np.exp(-g)) * u


def rmsnorm(x, eps=1e-5):
    """x / sqrt(mean(x^2) + eps), unit weight (the pages do not describe the norm)."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def round_bf16(x):
    """Store a value as bfloat16 the way a float32 kernel result is stored.

    First round to float32 (the kernels' accumulator type), then to the
    nearest bfloat16 with ties to even.  Returned as float64.
    """
    x32 = np.asarray(x, np.float64).astype(np.float32)
    bits = x32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(x32)
    out = rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(nan, np.nan, out)


# ---------------------------------------------------------------------------
# Outlier-smoothing rotations (WSVD page §2C: S1 on the activations and S2 on
# the latent, both orthogonal, applied before RTN; LASER page §3: a rotation
# between the SVD factors before quantisation).  Orthogonal maps do not change
# what is computed -- x A = (x S1)(S1^T A), c B = (c S2)(S2^T B) -- only which
# values get quantised.  Readings: S1 is the normalised Walsh-Hadamard matrix
# of the activation width (a power of two); S2 is block diagonal, each block
# the normalised Walsh-Hadamard matrix of order n = the largest power of two
# dividing r (at most 64).
# ---------------------------------------------------------------------------

def hadamard(n):
    """Normalised Walsh-Hadamard matrix of order n (a power of two), by
    Sylvester's doubling: H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]], then
    divided by sqrt(n).  Symmetric and orthogonal."""
    assert n >= 1 and (n & (n - 1)) == 0
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h / math.sqrt(n)


def latent_rotation(r):
    """S2 for an r-dim latent: block diagonal with blocks hadamard(n), n the
    largest power of two dividing r, capped at 64."""
    n = 1
    while r % (2 * n) == 0 and 2 * n <= 64:
        n *= 2
    s2 = np.zeros((r, r))
    for b0 in range(0, r, n):
        s2[b0:b0 + n, b0:b0 + n] = hadamard(n)
    return s2


def rotate_latents(v, ranks):
    """Each head's latent v^h (consecutive blocks of v [..., sum ranks]) times
    its S2, in float64, rounded once to float32 (what gets quantised)."""
    v = np.asarray(v, np.float64)
    out = np.empty_like(v)
    off = 0
    for r in ranks:
        out[..., off:off + r] = v[..., off:off + r] @ latent_rotation(r)
        off += r
    return out.astype(np.float32)


def rmsnorm_hadamard(x, eps=1e-5):
    """S1 after the pre-norm: RMSNorm(x) times hadamard(k), k = the row width."""
    x = rmsnorm(x, eps)
    return x @ hadamard(x.shape[-1])


# ---------------------------------------------------------------------------
# Rotary positions (an extension: neither page mentions positional encoding).
# The WSVD page's fused kernel rebuilds K_h on chip from the latent (§2C);
# with a rotary position encoding that rebuild is required, since the
# rotation of each key depends on its position and q can no longer be folded
# into B_K.  Readings: rotate-half pairs (dim i with dim i + H/2), frequencies
# theta_i = base^(-2 i / H) with base 10000, keys at their cache positions
# 0 .. len - 1, the query at the position of the newest cached token
# (len - 1), values not rotated (so V keeps the latent form).
# ---------------------------------------------------------------------------

def rope_angles(positions, H, base=10000.0):
    """angle[t, i] = positions[t] * base^(-2 i / H) for i < H / 2 (float64)."""
    i = np.arange(H // 2, dtype=np.float64)
    theta = float(base) ** (-2.0 * i / H)
    return np.asarray(positions, np.float64)[:, None] * theta[None, :]


def rope(x, positions, base=10000.0):
    """Rotate-half rotary encoding of rows x [T, H] at positions [T]: for each
    i < H/2 the pair (x_i, x_{i+H/2}) is turned by angle[t, i]."""
    x = np.asarray(x, np.float64)
    H = x.shape[-1]
    h = H // 2
    ang = rope_angles(positions, H, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :h], x[:, h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def attention_rope(q, Ck_hat, Cv_hat, B_K, B_V, softmax_scale, q_pos, base=10000.0, k_pos0=0):
    """Attention of one (batch, head) with rotary keys and query.

    K = Ck_hat B_K rebuilt, each row t rotated at position k_pos0 + t; q
    rotated at q_pos; s = K_rot q_rot * scale; o = softmax(s) (Cv_hat B_V).
    """
    K = np.asarray(Ck_hat, np.float64) @ np.asarray(B_K, np.float64)   # rebuilt keys [T, H]
    V = np.asarray(Cv_hat, np.float64) @ np.asarray(B_V, np.float64)   # values [T, H]
    T = K.shape[0]
    K_rot = rope(K, k_pos0 + np.arange(T), base)
    q_rot = rope(np.asarray(q, np.float64)[None, :], [q_pos], base)[0]
    s = (K_rot @ q_rot) * float(softmax_scale)
    s = s - np.max(s)
    p = np.exp(s)
    p = p / np.sum(p)
    return p @ V


def latent_attention_rope(q, cache_k, cache_v, B_K_heads, B_V_heads, softmax_scale, base=10000.0):
    """attention_rope for every (b, h) over the whole cache; the query of row
    b sits at position len_b - 1.  Returns o: [B, n_h, H] float64."""
    q = np.asarray(q, np.float64)
    Bsz, n_h, H = q.shape
    out = np.zeros((Bsz, n_h, H), np.float64)
    for b in range(Bsz):
        T = cache_k.length(b)
        if T == 0:
            continue
        for h in range(n_h):
            out[b, h] = attention_rope(q[b, h], cache_k.dequant(b, h), cache_v.dequant(b, h),
                                       B_K_heads[h], B_V_heads[h], softmax_scale, T - 1, base)
    return out


# ---------------------------------------------------------------------------
# Per-head truncated SVD (WSVD page §2A), used to build factors from dense heads
# ---------------------------------------------------------------------------

def per_head_svd(W_head, r):
    """Rank-r truncated SVD of one head's E x H projection slice.

    Returns (A [E, r], B [r, H]) with A = U_r diag(sigma_r), B = V_r^T, so that
    x W ~ (x A) B and x A is the per-head latent that gets cached.
    """
    W = np.asarray(W_head, np.float64)
    U, sig, Vt = np.linalg.svd(W, full_matrices=False)
    return U[:, :r] * sig[None, :r], Vt[:r, :]


# ---------------------------------------------------------------------------
# One W8A8 decoder-layer decode step (pre-norm block; composition is a reading)
# ---------------------------------------------------------------------------

def _linear_dense_w8a8(x_q, x_scale, W, s_W, residual=None):
    k_in = np.asarray(W).shape[0]
    y, _, _ = linear_w8a8_hybrid(x_q, x_scale, np.arange(k_in), np.zeros(0, np.int64),
                                 W, s_W, None, None, None, None, residual=residual)
    return y


def decoder_layer_w8a8(x, layer, cache_k, cache_v, eps=1e-5):
    """One decode step of a W8A8 pre-norm decoder layer with latent attention.

    x: [B, E] bf16 values (as float).  ``layer`` is a dict of int8 weights and
    fp16 scales: W_Q, s_Q, W_O, s_O, A (int8 [E, sum r_K + sum r_V]), s_A,
    B_K / B_V (lists of [r, H] bf16 values), ranks_k, ranks_v, n_heads,
    head_dim, and gate / up / down hybrid weights (dicts with dense_idx,
    lr_idx, W_D, s_D, U, s_U, V, s_V).  Each cache gets one appended token per
    batch row.  Every intermediate that the device path stores as bf16 is
    rounded to bf16 here at the same point; int8 activations are quantised
    from float32 values.  Returns the layer output [B, E] (float64, before the
    final bf16 rounding) and a dict of intermediates.
    """
    Bsz, E = x.shape
    n_h, H = layer["n_heads"], layer["head_dim"]
    x = np.asarray(x, np.float64)
    h1 = rmsnorm(x, eps).astype(np.float32)
    xq, sx = quantize_rows_i8(h1)
    q = round_bf16(_linear_dense_w8a8(xq, sx, layer["W_Q"], layer["s_Q"]))
    v = latent_project_w8a8(xq, sx, layer["A"], layer["s_A"])
    rk, rv = layer["ranks_k"], layer["ranks_v"]
    nk = int(np.sum(rk))
    qk = quantize_latents(v[:, :nk], rk, "i8", 32)
    qv = quantize_latents(v[:, nk:], rv, "i8", 32)
    for b in range(Bsz):
        cache_k.append(b, [(c[b:b + 1], s[b:b + 1]) for c, s in qk])
        cache_v.append(b, [(c[b:b + 1], s[b:b + 1]) for c, s in qv])
    attn = latent_attention(q.reshape(Bsz, n_h, H), cache_k, cache_v,
                            layer["B_K"], layer["B_V"], 1.0 / math.sqrt(H))
    attn = round_bf16(attn.reshape(Bsz, n_h * H))
    aq, sa = quantize_rows_i8(attn.astype(np.float32))
    x2 = round_bf16(_linear_dense_w8a8(aq, sa, layer["W_O"], layer["s_O"], residual=x))
    h2 = rmsnorm(x2, eps).astype(np.float32)
    hq, sh = quantize_rows_i8(h2)
    g = layer["gate"]
    u = layer["up"]
    gate, _, _ = linear_w8a8_hybrid(hq, sh, g["dense_idx"], g["lr_idx"], g["W_D"], g["s_D"],
                                    g["U"], g["s_U"], g["V"], g["s_V"])
    upv, _, _ = linear_w8a8_hybrid(hq, sh, u["dense_idx"], u["lr_idx"], u["W_D"], u["s_D"],
                                   u["U"], u["s_U"], u["V"], u["s_V"])
    gate = round_bf16(gate)
    upv = round_bf16(upv)
    act = swiglu(gate, upv).astype(np.float32)
    mq, sm = quantize_rows_i8(act)
    d = layer["down"]
    out, _, _ = linear_w8a8_hybrid(mq, sm, d["dense_idx"], d["lr_idx"], d["W_D"], d["s_D"],
                                   d["U"], d["s_U"], d["V"], d["s_V"], residual=x2)
    inter = dict(xq=xq, sx=sx, q=q, latent=v, attn=attn, aq=aq, sa=sa, x2=x2, hq=hq, sh=sh,
                 gate=gate, up=upv, mq=mq, sm=sm)
    return out, inter
