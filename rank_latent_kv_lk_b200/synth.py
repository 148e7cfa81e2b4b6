"""Seeded synthetic inputs for the decode workloads.

Random draws, dtype rounding and index sets only: no step of the decode
method is computed here.  The same functions feed the library (tests, bench)
and the CPU oracle (tests), so both see identical inputs.

Recipe (shapes from rank_latent_kv_lk_b200.configs):
  * hidden states x ~ N(0, 1); the first `image_tokens` positions of the
    context ~ N(0, image_sigma^2) ("image" tokens); a seeded set of
    outlier_frac of the channels is multiplied by outlier_scale;
  * latent factor A ~ N(0, 1/E) stored [sum r, E]; B_K^h, B_V^h ~ N(0, 1/r_h)
    stored [r_h, H] per head; float workloads keep them in the activation
    dtype (fp32 or bf16);
  * queries q ~ N(0, 1) per decode step (the law of x W_Q with W_Q ~ N(0, 1/E));
  * W8A8 weights: int8 codes clamp(rint(40 z), -127, 127), z ~ N(0, 1), with
    per-output-channel fp16 scales 1 / (40 sqrt(fan_in)) * U(0.8, 1.2);
  * ranks drawn per (layer, head) from rank_choices, K and V independently.
Every draw uses a torch.Generator seeded from (workload seed, purpose, layer).
Bulk context tokens of the large workloads are drawn on the GPU with torch's
device generator (same seeding rule); everything else on the CPU.
"""
from __future__ import annotations

import math

import numpy as np
import torch

RANKS, FACTORS, CONTEXT, DECODE, QUERIES, OUTLIERS, WEIGHTS = range(7)

_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "i8": torch.bfloat16}


def seed_for(w, purpose, layer=0):
    return (w.seed * 100003 + purpose * 1009 + layer) % (2 ** 63)


def generator(w, purpose, layer=0, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(seed_for(w, purpose, layer))
    return g


def act_dtype(w):
    return _DT[w.act]


def bulk_device(w):
    """Where context tokens are drawn: the GPU for workloads too large for a quick CPU draw."""
    return "cuda" if w.batch * w.context * w.embed_dim > (1 << 26) else "cpu"


def ranks(w):
    """(ranks_k, ranks_v): lists over layers of lists over heads."""
    if w.rank:
        rk = [[w.rank] * w.n_heads for _ in range(w.n_layers)]
        return rk, [list(r) for r in rk]
    g = generator(w, RANKS)
    ch = torch.tensor(w.rank_choices)
    ik = torch.randint(len(w.rank_choices), (w.n_layers, w.n_heads), generator=g)
    iv = torch.randint(len(w.rank_choices), (w.n_layers, w.n_heads), generator=g)
    return ch[ik].tolist(), ch[iv].tolist()


def outlier_channels(w):
    if w.outlier_frac <= 0:
        return None
    g = generator(w, OUTLIERS)
    n = int(round(w.outlier_frac * w.embed_dim))
    return torch.sort(torch.randperm(w.embed_dim, generator=g)[:n]).values


def factors(w, layer, ranks_k, ranks_v):
    """Float latent factors for one layer: A [sum r_K + sum r_V, E], B_K [sum r_K, H], B_V [sum r_V, H]."""
    g = generator(w, FACTORS, layer)
    dt = act_dtype(w)
    n_tot = sum(ranks_k) + sum(ranks_v)
    A = (torch.randn(n_tot, w.embed_dim, generator=g) / math.sqrt(w.embed_dim)).to(dt)
    BK = torch.cat([torch.randn(r, w.head_dim, generator=g) / math.sqrt(r) for r in ranks_k]).to(dt)
    BV = torch.cat([torch.randn(r, w.head_dim, generator=g) / math.sqrt(r) for r in ranks_v]).to(dt)
    return A, BK, BV


def int8_weight(g, n_out, k_in):
    """int8 codes [n_out, k_in] and fp16 per-output scales [n_out]."""
    codes = torch.clamp(torch.round(torch.randn(n_out, k_in, generator=g) * 40.0), -127, 127).to(torch.int8)
    scale = (torch.rand(n_out, generator=g) * 0.4 + 0.8) / (40.0 * math.sqrt(k_in))
    return codes, scale.to(torch.float16)


def _shape_tokens(w, x, pos0):
    """Apply the image-token sigma and the outlier channels to N(0,1) draws x [B, n, E]."""
    n = x.shape[1]
    if w.image_tokens and pos0 < w.image_tokens:
        k = min(n, w.image_tokens - pos0)
        x[:, :k] *= w.image_sigma
    ch = outlier_channels(w)
    if ch is not None:
        x[:, :, ch.to(x.device)] *= w.outlier_scale
    return x


def context_tokens(w, layer=0, device=None):
    """Context hidden states [B, context, E] in the activation dtype (bf16 for W8A8 layers)."""
    device = device or bulk_device(w)
    g = generator(w, CONTEXT, layer, device=device)
    x = torch.randn(w.batch, w.context, w.embed_dim, generator=g, device=device)
    return _shape_tokens(w, x, 0).to(act_dtype(w))


def decode_tokens(w, layer=0):
    """Hidden states of the decode steps [steps, B, E] (CPU)."""
    g = generator(w, DECODE, layer)
    x = torch.randn(w.steps, w.batch, w.embed_dim, generator=g)
    x = _shape_tokens(w, x.transpose(0, 1), w.context).transpose(0, 1)
    return x.contiguous().to(act_dtype(w))


def queries(w, layer=0):
    """Queries [steps, B, n_heads, H] (CPU), for workloads whose q is an input."""
    g = generator(w, QUERIES, layer)
    return torch.randn(w.steps, w.batch, w.n_heads, w.head_dim, generator=g).to(act_dtype(w))


def layer_weights_w8a8(w, ranks_k, ranks_v):
    """Weights of one W8A8 decoder layer (CPU): W_Q, W_O, A (int8 + fp16 scales),
    B_K / B_V (bf16) and the hybrid gate / up / down projections."""
    g = generator(w, WEIGHTS)
    E, nh, H = w.embed_dim, w.n_heads, w.head_dim
    out = {}
    out["W_Q"], out["s_Q"] = int8_weight(g, nh * H, E)
    out["W_O"], out["s_O"] = int8_weight(g, E, nh * H)
    n_tot = sum(ranks_k) + sum(ranks_v)
    out["A"], out["s_A"] = int8_weight(g, n_tot, E)
    out["B_K"] = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(torch.bfloat16)
    out["B_V"] = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(torch.bfloat16)
    for name, (k_in, n_out) in (("gate", (E, w.ffn_inter)), ("up", (E, w.ffn_inter)),
                                ("down", (w.ffn_inter, E))):
        n_dense = int(round(w.ffn_dense_frac * k_in / 16)) * 16
        perm = torch.randperm(k_in, generator=g)
        D = torch.sort(perm[:n_dense]).values.to(torch.int32)
        notD = torch.sort(perm[n_dense:]).values.to(torch.int32)
        W_D, s_D = int8_weight(g, n_out, n_dense)
        U, s_U = int8_weight(g, w.ffn_rank, k_in - n_dense)
        V, s_V = int8_weight(g, n_out, w.ffn_rank)
        out[name] = dict(dense_idx=D, lr_idx=notD, W_D=W_D, s_D=s_D, U=U, s_U=s_U, V=V, s_V=s_V)
    return out


def ffn_outsplit_weights(w, k_in=None, n_out=None, rank=None, dense_frac=None, seed_purpose=None):
    """Gate and up weights of the FFN split on output channels (CPU), with the
    workload's int8 recipe: a seeded dense_frac of the hidden channels (a
    multiple of 16) keep dense rows W_D [n_dense, k_in], the others come from
    U [rank, k_in] and V [n_out - n_dense, rank].  Gate and up share the split."""
    g = generator(w, WEIGHTS if seed_purpose is None else seed_purpose)
    k_in = w.embed_dim if k_in is None else k_in
    n_out = w.ffn_inter if n_out is None else n_out
    rank = w.ffn_rank if rank is None else rank
    frac = w.ffn_dense_frac if dense_frac is None else dense_frac
    n_dense = int(round(frac * n_out / 16)) * 16
    perm = torch.randperm(n_out, generator=g)
    dense_out = torch.sort(perm[:n_dense]).values.to(torch.int32)
    lr_out = torch.sort(perm[n_dense:]).values.to(torch.int32)
    out = dict(dense_out=dense_out, lr_out=lr_out, k_in=k_in, n_out=n_out, rank=rank, n_dense=n_dense)
    for name in ("gate", "up"):
        W_D, s_D = int8_weight(g, n_dense, k_in)
        U, s_U = int8_weight(g, rank, k_in)
        V, s_V = int8_weight(g, n_out - n_dense, rank)
        out[name] = dict(W_D=W_D, s_D=s_D, U=U, s_U=s_U, V=V, s_V=s_V)
    return out


def as_numpy(t):
    """Exact host copy of a tensor as numpy (bf16 values widened to float32)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.to(torch.float32)
    return t.numpy()


def random_latents(shape, seed, sigma=1.3):
    """Latent values for quantiser and attention unit cases (float32, CPU)."""
    g = torch.Generator()
    g.manual_seed(seed)
    return (torch.randn(*shape, generator=g) * sigma).numpy().astype(np.float32)
