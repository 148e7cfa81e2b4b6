"""Per-head latent-KV decode on B200 (sm_100a): a C-ABI CUDA library plus thin
torch wrappers.  See include/lk.h for the boundary."""
from .api import (LatentCache, LowrankWeight, device_status, latent_decode_attn, latent_decode_step,  # noqa: F401
                  latent_project_append, lowrank_linear, quantize_latent, quantize_rows_i8,
                  rmsnorm_quant_i8, swiglu_quant_i8, workspaces)
from ._lib import LkError  # noqa: F401
