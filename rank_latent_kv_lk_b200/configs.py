"""The five decode workloads (LLaVA-class shapes from the WSVD and LASER pages).

Shapes only; inputs are drawn by rank_latent_kv_lk_b200.synth.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    key: int
    name: str
    n_layers: int
    batch: int
    embed_dim: int
    n_heads: int
    head_dim: int
    rank: int = 0                   # uniform rank for K and V (0: drawn per head)
    rank_choices: tuple = ()        # ranks drawn per (layer, head), K and V independently
    kind: str = "i8"                # latent codes: 'i8' (fp32 scale) or 'i4' (fp16 group scale)
    group: int = 32                 # int4 group size along r (effective min(group, r))
    act: str = "bf16"               # activations / factors: 'f32', 'bf16' or 'i8' (W8A8)
    context: int = 256              # tokens already in the cache
    steps: int = 1                  # decode steps, each appends one token per row
    image_tokens: int = 0           # leading "image" tokens drawn with image_sigma
    image_sigma: float = 1.0
    outlier_frac: float = 0.0       # fraction of x channels scaled by outlier_scale
    outlier_scale: float = 1.0
    ffn_inter: int = 0              # hybrid FFN intermediate size (full layer only)
    ffn_dense_frac: float = 0.0     # fraction of input channels kept dense
    ffn_rank: int = 0
    seed: int = 0

    @property
    def capacity(self):
        n = self.context + self.steps
        return (n + 15) // 16 * 16


WORKLOADS = {
    1: Workload(1, "single-layer fp32: E=512, 8x64 heads, r=16, B=1, T=256+1", 1, 1, 512, 8, 64,
                rank=16, act="f32", context=256, steps=1, seed=1001),
    2: Workload(2, "llava7b-attn: E=4096, 32x128 heads, r=32 int8, B=1, T=4096, 128 steps", 1, 1, 4096, 32,
                128, rank=32, context=4096, steps=128, image_tokens=576, image_sigma=1.5, seed=1002),
    3: Workload(3, "llava7b-attn: E=4096, 32x128 heads, r=24 int4 g32, B=16, T=8192, 128 steps, 5% x20 outliers",
                1, 16, 4096, 32, 128, rank=24, kind="i4", group=32, context=8192, steps=128, image_tokens=576,
                image_sigma=1.5, outlier_frac=0.05, outlier_scale=20.0, seed=1003),
    4: Workload(4, "laser-ragged: 32 layers x 32x128 heads, r in {8,16,32,48,64}, int8, B=8, T=16384+1",
                32, 8, 4096, 32, 128, rank_choices=(8, 16, 32, 48, 64), context=16384, steps=1, seed=1004),
    5: Workload(5, "w8a8 decoder layer: E=4096, 32x128 heads, r=32 int8, B=32, T=4096+1, hybrid FFN I=11008",
                1, 32, 4096, 32, 128, rank=32, act="i8", context=4096, steps=1, ffn_inter=11008,
                ffn_dense_frac=0.25, ffn_rank=512, seed=1005),
}
