"""Per-head latent-KV decode on B200 (sm_100a): a C-ABI CUDA library plus thin
torch wrappers.  See include/lk.h for the boundary.

The library (liblk.so) is loaded on first use of a wrapper, so the input
generators (``synth``, ``configs``) import without it; every wrapper still
fails loudly when the library is missing."""
import importlib

_API = ("LatentCache", "LowrankWeight", "device_status", "latent_decode_attn", "latent_decode_step",
        "latent_project_append", "lowrank_linear", "quantize_latent", "quantize_rows_i8", "rmsnorm_quant_i8",
        "rmsnorm_hadamard_quant_i8", "swiglu_quant_i8", "workspaces", "kernel_launches", "dense_decode_attn", "reconstruct_kv",
        "rope_table", "latent_decode_attn_rope", "OutsplitFfn")


def __getattr__(name):
    if name in _API:
        return getattr(importlib.import_module(".api", __name__), name)
    if name == "LkError":
        return importlib.import_module("._lib", __name__).LkError
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


__all__ = list(_API) + ["LkError"]
