"""One W8A8 pre-norm decoder layer with latent attention and LASER hybrid FFN.

Composition (the pages do not describe the block; a LLaMA-style pre-norm
layer with unit RMSNorm weights, eps 1e-5, no positional rotation):

  x_q      = int8(RMSNorm(x))
  q        = x_q W_Q^T                      (W8A8 dense linear)
  latents  = quant(x_q A^T) appended        (lk_latent_decode_step: append,
  a        = latent attention                 then attention)
  x2       = x + int8(a) W_O^T              (W8A8 dense linear + residual)
  h_q      = int8(RMSNorm(x2))
  g, u     = hybrid(h_q; gate), hybrid(h_q; up)     (LASER hybrid linear)
  m_q      = int8(silu(g) * u)
  out      = x2 + hybrid(m_q; down)

Every step is a call into the C ABI; this module only wires buffers.
"""
from __future__ import annotations

import torch

from .api import (LatentCache, LowrankWeight, latent_decode_step, lowrank_linear, quantize_rows_i8,
                  rmsnorm_quant_i8, swiglu_quant_i8)


def dense_weight(W, s, device):
    """A plain W8A8 linear as a hybrid linear whose every input channel is dense."""
    n_out, k_in = W.shape
    idx = torch.arange(k_in, dtype=torch.int32, device=device)
    return LowrankWeight(k_in, n_out, 0, idx, None, W.to(device), s.to(device), None, None, None, None)


def hybrid_weight(d, k_in, n_out, device):
    t = {k: v.to(device) for k, v in d.items()}
    return LowrankWeight(k_in, n_out, int(t["U"].shape[0]), t["dense_idx"], t["lr_idx"], t["W_D"], t["s_D"],
                         t["U"], t["s_U"], t["V"], t["s_V"])


class W8A8DecoderLayer:
    def __init__(self, weights, n_heads, head_dim, ranks_k, ranks_v, batch, capacity, ffn_inter,
                 device="cuda"):
        E = weights["W_Q"].shape[1]
        self.E, self.n_heads, self.head_dim = E, n_heads, head_dim
        self.batch = batch
        self.wq = dense_weight(weights["W_Q"], weights["s_Q"], device)
        self.wo = dense_weight(weights["W_O"], weights["s_O"], device)
        self.A = weights["A"].to(device)
        self.s_A = weights["s_A"].to(device)
        self.B_K = weights["B_K"].to(device)
        self.B_V = weights["B_V"].to(device)
        self.gate = hybrid_weight(weights["gate"], E, ffn_inter, device)
        self.up = hybrid_weight(weights["up"], E, ffn_inter, device)
        self.down = hybrid_weight(weights["down"], ffn_inter, E, device)
        self.cache_k = LatentCache(batch, ranks_k, capacity, "i8", 32, device)
        self.cache_v = LatentCache(batch, ranks_v, capacity, "i8", 32, device, role="v")

    def step(self, x, seq_len, lens, trace=None):
        """x: [B, E] bf16 (device); seq_len: device int32 [B]; lens: host list (advanced in place).

        If `trace` is a dict, the intermediate device tensors are stored in it."""
        B = x.shape[0]
        xq, sx = rmsnorm_quant_i8(x)
        q = lowrank_linear(self.wq, xq, sx)
        # append the new token's latents, then attend (the attention launch
        # overlaps the append)
        attn = latent_decode_step(self.cache_k, self.cache_v, xq, self.A, seq_len, lens,
                                  q.view(B, self.n_heads, self.head_dim), self.B_K, self.B_V, x_scale=sx,
                                  a_scale=self.s_A, out_dtype=torch.bfloat16)
        for b in range(B):
            lens[b] += 1
        aq, sa = quantize_rows_i8(attn.view(B, self.n_heads * self.head_dim))
        x2 = lowrank_linear(self.wo, aq, sa, residual=x)
        hq, sh = rmsnorm_quant_i8(x2)
        g = lowrank_linear(self.gate, hq, sh)
        u = lowrank_linear(self.up, hq, sh)
        mq, sm = swiglu_quant_i8(g, u)
        out = lowrank_linear(self.down, mq, sm, residual=x2)
        if trace is not None:
            trace.update(xq=xq, sx=sx, q=q, attn=attn, aq=aq, sa=sa, x2=x2, hq=hq, sh=sh, gate=g, up=u, mq=mq,
                         sm=sm, out=out)
        return out
