"""Thin torch-facing wrappers over the C ABI (marshalling only).

Tensors are device tensors allocated by torch; the library computes.  Every
wrapper raises LkError when the library rejects its arguments.
"""
from __future__ import annotations

import ctypes as C
import math

import torch

from ._lib import (LK_BF16, LK_F16, LK_F32, LK_I4, LK_I8, LatentCacheDesc, LowrankWeightDesc, OutsplitWeightDesc,
                   check, lib)
from .layout import CacheGeometry

_DT = {torch.float32: LK_F32, torch.bfloat16: LK_BF16, torch.float16: LK_F16, torch.int8: LK_I8}


def _dtype_code(t):
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


class _WorkspacePool:
    """Zero-initialised per-device scratch buffers, one per purpose.

    Each entry point keeps its own buffer because the arrival counters at the
    start of a workspace must read zero at the start of every call (every
    completed call leaves them zero)."""

    def __init__(self):
        self._bufs = {}

    def get(self, purpose, nbytes, device):
        key = (purpose, str(device))
        buf = self._bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            self._bufs[key] = buf
        return buf


workspaces = _WorkspacePool()


class LatentCache:
    """Device latent cache of one layer for K or V (codes + scales planes)."""

    def __init__(self, batch, ranks, capacity, kind="i8", group=32, device="cuda", role="k", rotation=False):
        """role: 'k' or 'v' -- the two caches of a layer lay codes out differently.
        rotation: the append multiplies each head's latent by its block-Hadamard
        S2 before quantising (decode then takes the factors S2 B)."""
        if kind not in ("i8", "i4"):
            raise ValueError("kind must be 'i8' or 'i4'")
        self.role = role
        self.geom = CacheGeometry(batch, ranks, capacity, kind, group, role)
        self.batch, self.ranks, self.capacity, self.kind, self.group = batch, list(ranks), capacity, kind, group
        self.codes = torch.zeros(self.geom.codes_bytes, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(self.geom.scales_elems,
                                  dtype=torch.float32 if kind == "i8" else torch.float16, device=device)
        self._ranks = (C.c_int32 * len(self.ranks))(*self.ranks)
        self._desc = LatentCacheDesc(batch, len(self.ranks), capacity, LK_I8 if kind == "i8" else LK_I4,
                                     group, self._ranks, self.codes.data_ptr(), self.scales.data_ptr(),
                                     1 if rotation else 0)
        self.rotation = bool(rotation)

    @property
    def n_heads(self):
        return len(self.ranks)

    def desc(self):
        return C.byref(self._desc)

    def load(self, rows, scales):
        """Fill from logical code rows (rows[b][h]: uint8 [T, rb]) and scales."""
        c, s = self.geom.pack(rows, scales)
        self.codes.copy_(torch.from_numpy(c))
        self.scales.copy_(torch.from_numpy(s))

    def read(self, lens):
        """Logical code rows and scales of the first lens[b] tokens (host copies)."""
        return self.geom.unpack(self.codes.cpu().numpy(), self.scales.cpu().numpy(), lens)

    def read_unit(self, b, h, T):
        """Code rows [T, rb_h] and scales of the first T tokens of one (b, h) (host copies)."""
        off, n = self.geom.code_plane(b, h)
        soff, sn = self.geom.scale_plane(b, h)
        return self.geom.unpack_unit(self.codes[off:off + n].cpu().numpy(),
                                     self.scales[soff:soff + sn].cpu().numpy(), h, T)


def latent_project_append(k_cache, v_cache, x, A, seq_len, seq_len_host, x_scale=None, a_scale=None,
                          stream=None):
    """Project new tokens to per-head latents, quantise them and append.

    x: [B * n_new, E] (f32 / bf16 / int8); A: [sum r_K + sum r_V, E] same dtype;
    int8 inputs need x_scale fp32 [B * n_new] and a_scale fp16 [N_tot].
    seq_len: device int32 [B] (advanced by n_new); seq_len_host: list of ints.
    """
    rows = x.shape[0]
    if rows % k_cache.batch:
        raise ValueError("x rows must be a multiple of the batch")
    n_new = rows // k_cache.batch
    E = x.shape[-1]
    xdt = _dtype_code(x)
    host = (C.c_int32 * k_cache.batch)(*[int(v) for v in seq_len_host])
    need = lib.lk_latent_project_workspace_bytes(k_cache.desc(), v_cache.desc(), E, n_new, xdt)
    ws = workspaces.get("project", need, x.device)
    check(lib.lk_latent_project_append(
        k_cache.desc(), v_cache.desc(), _ptr(x), xdt, _ptr(x_scale), _ptr(A), _dtype_code(A), _ptr(a_scale),
        E, n_new, _ptr(seq_len), host, _ptr(ws), ws.numel(), _stream(stream)))


def latent_decode_attn(k_cache, v_cache, q, B_K, B_V, seq_len, max_seq_len, softmax_scale=None, out=None,
                       out_dtype=None, n_split=0, stream=None):
    """softmax(q K^T * scale) V over the latent caches, without forming K or V.

    q: [B, n_heads, H]; B_K / B_V: per-head factors packed head after head,
    [sum r, H]; seq_len: device int32 [B]; max_seq_len: host bound.
    """
    H = q.shape[-1]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(H)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    need = lib.lk_latent_decode_workspace_bytes(k_cache.desc(), v_cache.desc(), int(max_seq_len), int(n_split))
    # one buffer per B * n_heads: the counters at its start must read zero, and
    # the partials of another shape could cover them
    ws = workspaces.get(("decode", k_cache.batch * len(k_cache.ranks)), need, q.device)
    check(lib.lk_latent_decode_attn(
        k_cache.desc(), v_cache.desc(), _ptr(q), _dtype_code(q), _ptr(B_K), _ptr(B_V), _dtype_code(B_K), H,
        _ptr(seq_len), int(max_seq_len), float(softmax_scale), _ptr(out), _dtype_code(out), int(n_split),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out


def latent_decode_step(k_cache, v_cache, x, A, seq_len, seq_len_host, q, B_K, B_V, x_scale=None, a_scale=None,
                       softmax_scale=None, out=None, out_dtype=None, n_split=0, stream=None):
    """One decode step: append one token per row (x: [B, E]), then attend over
    the caches including it.  The attention launch overlaps the append (its
    q absorption runs while the append finishes).  seq_len (device) advances
    by one; seq_len_host is the host copy before the step."""
    H = q.shape[-1]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(H)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    E = x.shape[-1]
    xdt = _dtype_code(x)
    host = (C.c_int32 * k_cache.batch)(*[int(v) for v in seq_len_host])
    pneed = lib.lk_latent_project_workspace_bytes(k_cache.desc(), v_cache.desc(), E, 1, xdt)
    pws = workspaces.get("project", pneed, x.device)
    max_len = max(int(v) for v in seq_len_host) + 1
    dneed = lib.lk_latent_decode_workspace_bytes(k_cache.desc(), v_cache.desc(), max_len, int(n_split))
    dws = workspaces.get(("decode", k_cache.batch * len(k_cache.ranks)), dneed, q.device)
    check(lib.lk_latent_decode_step(
        k_cache.desc(), v_cache.desc(), _ptr(x), xdt, _ptr(x_scale), _ptr(A), _dtype_code(A), _ptr(a_scale), E,
        _ptr(seq_len), host, _ptr(q), _dtype_code(q), _ptr(B_K), _ptr(B_V), _dtype_code(B_K), H,
        float(softmax_scale), _ptr(out), _dtype_code(out), int(n_split), _ptr(pws), pws.numel(), _ptr(dws),
        dws.numel(), _stream(stream)))
    return out


def dense_decode_attn(q, K, V, seq_len, max_seq_len, softmax_scale=None, out=None, out_dtype=None, stream=None):
    """Dense bf16 flash-decoding over materialised K, V [B, heads, capacity, H] (comparison point)."""
    B, nh, cap, H = K.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(H)
    if out is None:
        out = torch.empty((B, nh, H), dtype=out_dtype or q.dtype, device=q.device)
    need = lib.lk_dense_decode_workspace_bytes(B, nh, H, int(max_seq_len))
    ws = workspaces.get(("dense", B * nh), need, q.device)
    check(lib.lk_dense_decode_attn(_ptr(q), _ptr(K), _ptr(V), B, nh, H, cap, _ptr(seq_len), int(max_seq_len),
                                   float(softmax_scale), _ptr(out), _dtype_code(out), _ptr(ws), ws.numel(),
                                   _stream(stream)))
    return out


class OutsplitFfn:
    """Device gate and up weights of the FFN split on output channels (int8,
    fp16 scales; see lk_ffn_gate_up_swiglu).  d: a dict as from
    synth.ffn_outsplit_weights."""

    def __init__(self, d, device="cuda"):
        self.k_in, self.n_out, self.rank, self.n_dense = d["k_in"], d["n_out"], d["rank"], d["n_dense"]
        self.dense_out = d["dense_out"].to(device)
        self.lr_out = d["lr_out"].to(device)
        self._keep = []
        self._desc = []
        for name in ("gate", "up"):
            t = {k: v.to(device) for k, v in d[name].items()}
            self._keep.append(t)
            self._desc.append(OutsplitWeightDesc(*[t[k].data_ptr() if t[k].numel() else None
                                                   for k in ("W_D", "s_D", "U", "s_U", "V", "s_V")]))

    def __call__(self, x_q, x_scale, out=None, stream=None):
        """silu(gate(x)) * up(x): fp32 [m, n_out]."""
        m = x_q.shape[0]
        if out is None:
            out = torch.empty((m, self.n_out), dtype=torch.float32, device=x_q.device)
        need = lib.lk_ffn_gate_up_swiglu_workspace_bytes(self.rank, m)
        ws = workspaces.get("ffn_outsplit", need, x_q.device)
        check(lib.lk_ffn_gate_up_swiglu(C.byref(self._desc[0]), C.byref(self._desc[1]), self.k_in, self.n_out,
                                        self.n_dense, self.rank, _ptr(self.dense_out), _ptr(self.lr_out),
                                        _ptr(x_q), _ptr(x_scale), m, _ptr(out), _ptr(ws), ws.numel(),
                                        _stream(stream)))
        return out


def rope_table(head_dim, max_pos, base=10000.0, device="cuda", stream=None):
    """cos / sin of t * base^(-2 i / head_dim): fp32 [max_pos, head_dim / 2, 2]."""
    table = torch.empty((max_pos, head_dim // 2, 2), dtype=torch.float32, device=device)
    check(lib.lk_rope_table(int(head_dim), int(max_pos), float(base), _ptr(table), _stream(stream)))
    return table


def latent_decode_attn_rope(k_cache, v_cache, q, B_K, B_V, seq_len, max_seq_len, table, softmax_scale=None,
                            out=None, out_dtype=None, stream=None):
    """Decode attention with rotary keys and query: keys rebuilt from the latent
    codes on chip and rotated at their positions, the query at the newest
    position (seq_len - 1); values in latent form.  B_K / B_V bf16."""
    H = q.shape[-1]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(H)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    need = lib.lk_latent_decode_rope_workspace_bytes(k_cache.desc(), v_cache.desc(), H, int(max_seq_len))
    ws = workspaces.get(("rope", k_cache.batch * len(k_cache.ranks)), need, q.device)
    check(lib.lk_latent_decode_attn_rope(
        k_cache.desc(), v_cache.desc(), _ptr(q), _dtype_code(q), _ptr(B_K), _ptr(B_V), _dtype_code(B_K), H,
        _ptr(seq_len), int(max_seq_len), _ptr(table), float(softmax_scale), _ptr(out), _dtype_code(out),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out


def reconstruct_kv(k_cache, v_cache, B_K, B_V, seq_len, max_seq_len, head_dim, K_out=None, V_out=None, stream=None):
    """The naive path: K, V rebuilt from the latent cache into bf16 [B, heads, capacity, H]."""
    shape = (k_cache.batch, len(k_cache.ranks), k_cache.capacity, head_dim)
    if K_out is None:
        K_out = torch.zeros(shape, dtype=torch.bfloat16, device=B_K.device)
    if V_out is None:
        V_out = torch.zeros(shape, dtype=torch.bfloat16, device=B_K.device)
    check(lib.lk_latent_reconstruct_kv(k_cache.desc(), v_cache.desc(), _ptr(B_K), _ptr(B_V), _dtype_code(B_K),
                                       head_dim, _ptr(seq_len), int(max_seq_len), _ptr(K_out), _ptr(V_out),
                                       _stream(stream)))
    return K_out, V_out


class LowrankWeight:
    """Device weights of one LASER hybrid linear (int8, fp16 scales)."""

    def __init__(self, k_in, n_out, rank, dense_idx, lr_idx, W_D, s_D, U, s_U, V, s_V):
        self.k_in, self.n_out, self.rank = k_in, n_out, rank
        self.n_dense = 0 if dense_idx is None else int(dense_idx.numel())
        self.tensors = (dense_idx, lr_idx, W_D, s_D, U, s_U, V, s_V)
        self._desc = LowrankWeightDesc(k_in, n_out, rank, self.n_dense, *[
            (t.data_ptr() if t is not None else None) for t in self.tensors])

    def desc(self):
        return C.byref(self._desc)


def lowrank_linear(w, x_q, x_scale, residual=None, y=None, y_dtype=torch.bfloat16, t_q_out=None, t_scale_out=None,
                   stream=None):
    m = x_q.shape[0]
    if y is None:
        y = torch.empty((m, w.n_out), dtype=y_dtype, device=x_q.device)
    need = lib.lk_lowrank_workspace_bytes(w.desc(), m)
    ws = workspaces.get("lowrank", need, x_q.device)
    check(lib.lk_lowrank_linear(w.desc(), _ptr(x_q), _ptr(x_scale), m, _ptr(residual), _ptr(y), _dtype_code(y),
                                _ptr(t_q_out), _ptr(t_scale_out), _ptr(ws), ws.numel(), _stream(stream)))
    return y


def quantize_latent(v, kind="i8", group=32, stream=None):
    """v: fp32 [m, r] -> (codes, scales) with the cache's quantisation rule."""
    m, r = v.shape
    if kind == "i8":
        codes = torch.empty((m, r), dtype=torch.int8, device=v.device)
        scales = torch.empty((m,), dtype=torch.float32, device=v.device)
    else:
        g = min(group, r)
        codes = torch.empty((m, r // 2), dtype=torch.uint8, device=v.device)
        scales = torch.empty((m, -(-r // g)), dtype=torch.float16, device=v.device)
    check(lib.lk_quantize_latent(_ptr(v), m, r, LK_I8 if kind == "i8" else LK_I4, group, _ptr(codes),
                                 _ptr(scales), _stream(stream)))
    return codes, scales


def quantize_rows_i8(x, stream=None):
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    s = torch.empty((m,), dtype=torch.float32, device=x.device)
    check(lib.lk_quantize_rows_i8(_ptr(x), _dtype_code(x), m, k, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def rmsnorm_quant_i8(x, eps=1e-5, stream=None):
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    s = torch.empty((m,), dtype=torch.float32, device=x.device)
    check(lib.lk_rmsnorm_quant_i8(_ptr(x), _dtype_code(x), m, k, float(eps), _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def rmsnorm_hadamard_quant_i8(x, eps=1e-5, stream=None):
    """RMSNorm, then the normalised Walsh-Hadamard transform of each row (S1),
    then per-row int8 quantisation; the row width must be a power of two."""
    m, k = x.shape
    q = torch.empty((m, k), dtype=torch.int8, device=x.device)
    s = torch.empty((m,), dtype=torch.float32, device=x.device)
    check(lib.lk_rmsnorm_hadamard_quant_i8(_ptr(x), _dtype_code(x), m, k, float(eps), _ptr(q), _ptr(s),
                                           _stream(stream)))
    return q, s


def swiglu_quant_i8(gate, up, stream=None):
    m, n = gate.shape
    q = torch.empty((m, n), dtype=torch.int8, device=gate.device)
    s = torch.empty((m,), dtype=torch.float32, device=gate.device)
    check(lib.lk_swiglu_quant_i8(_ptr(gate), _ptr(up), _dtype_code(gate), m, n, _ptr(q), _ptr(s),
                                 _stream(stream)))
    return q, s


def device_status(reset=True):
    """Synchronise and raise if a kernel reported an expired bounded wait."""
    check(lib.lk_device_status(1 if reset else 0))


def kernel_launches():
    """Kernels the library has enqueued in this process so far (lk_kernel_launches)."""
    return int(lib.lk_kernel_launches())
