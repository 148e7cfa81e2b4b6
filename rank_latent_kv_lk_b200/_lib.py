"""ctypes binding of liblk.so (the C ABI declared in include/lk.h).

Argument marshalling only: every computation happens in the library's CUDA
kernels.  Importing this module fails loudly if the library is missing; there
is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblk.so")

LK_OK = 0
LK_ERR_INVALID_ARG = 1
LK_ERR_SHAPE = 2
LK_ERR_DTYPE = 3
LK_ERR_ALIGN = 4
LK_ERR_CAPACITY = 5
LK_ERR_UNSUPPORTED = 6
LK_ERR_WORKSPACE = 7
LK_ERR_CUDA = 8
LK_ERR_DEVICE = 9

LK_F32, LK_BF16, LK_F16, LK_I8, LK_I4 = 0, 1, 2, 3, 4

LK_MAX_HEADS = 128
LK_MAX_RANK = 64
LK_MAX_HEAD_DIM = 256


class LatentCacheDesc(C.Structure):
    _fields_ = [
        ("batch", C.c_int32),
        ("n_heads", C.c_int32),
        ("capacity", C.c_int32),
        ("code_dtype", C.c_int),
        ("group", C.c_int32),
        ("ranks", C.POINTER(C.c_int32)),
        ("codes", C.c_void_p),
        ("scales", C.c_void_p),
        ("rotation", C.c_int32),
    ]


class LowrankWeightDesc(C.Structure):
    _fields_ = [
        ("k_in", C.c_int32),
        ("n_out", C.c_int32),
        ("rank", C.c_int32),
        ("n_dense", C.c_int32),
        ("dense_idx", C.c_void_p),
        ("lr_idx", C.c_void_p),
        ("W_D", C.c_void_p),
        ("s_D", C.c_void_p),
        ("U", C.c_void_p),
        ("s_U", C.c_void_p),
        ("V", C.c_void_p),
        ("s_V", C.c_void_p),
    ]


class OutsplitWeightDesc(C.Structure):
    _fields_ = [
        ("W_D", C.c_void_p),
        ("s_D", C.c_void_p),
        ("U", C.c_void_p),
        ("s_U", C.c_void_p),
        ("V", C.c_void_p),
        ("s_V", C.c_void_p),
    ]


class LkError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{message} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m rank_latent_kv_lk_b200.build` "
            "(there is no fallback implementation)")
    lib = C.CDLL(LIB_PATH)
    P = C.c_void_p
    I32 = C.c_int32
    SZ = C.c_size_t
    CP = C.POINTER(LatentCacheDesc)
    WP = C.POINTER(LowrankWeightDesc)
    sig = {
        "lk_version": (I32, []),
        "lk_kernel_launches": (C.c_uint64, []),
        "lk_last_error": (C.c_char_p, []),
        "lk_status_string": (C.c_char_p, [C.c_int]),
        "lk_latent_cache_bytes": (C.c_int, [CP, C.POINTER(SZ), C.POINTER(SZ)]),
        "lk_latent_project_append": (C.c_int, [CP, CP, P, C.c_int, P, P, C.c_int, P, I32, I32, P, P, P, SZ, P]),
        "lk_latent_project_workspace_bytes": (SZ, [CP, CP, I32, I32, C.c_int]),
        "lk_latent_decode_attn": (C.c_int, [CP, CP, P, C.c_int, P, P, C.c_int, I32, P, I32, C.c_float, P,
                                            C.c_int, I32, P, SZ, P]),
        "lk_latent_decode_workspace_bytes": (SZ, [CP, CP, I32, I32]),
        "lk_latent_decode_attn_noalloc": (C.c_int, [CP, CP, P, C.c_int, P, P, C.c_int, I32, P, I32, C.c_float, P,
                                                    C.c_int, I32, P]),
        "lk_debug_decode_attn_stall": (C.c_int, [CP, CP, P, C.c_int, P, P, C.c_int, I32, P, I32, C.c_float, P,
                                                 C.c_int, I32, P, SZ, I32, C.c_uint32, P]),
        "lk_latent_decode_step": (C.c_int, [CP, CP, P, C.c_int, P, P, C.c_int, P, I32, P, P, P, C.c_int, P, P,
                                            C.c_int, I32, C.c_float, P, C.c_int, I32, P, SZ, P, SZ, P]),
        "lk_dense_decode_attn": (C.c_int, [P, P, P, I32, I32, I32, I32, P, I32, C.c_float, P, C.c_int, P, SZ, P]),
        "lk_dense_decode_workspace_bytes": (SZ, [I32, I32, I32, I32]),
        "lk_latent_reconstruct_kv": (C.c_int, [CP, CP, P, P, C.c_int, I32, P, I32, P, P, P]),
        "lk_rope_table": (C.c_int, [I32, I32, C.c_float, P, P]),
        "lk_ffn_gate_up_swiglu": (C.c_int, [C.POINTER(OutsplitWeightDesc), C.POINTER(OutsplitWeightDesc), I32, I32,
                                            I32, I32, P, P, P, P, I32, P, P, SZ, P]),
        "lk_ffn_gate_up_swiglu_workspace_bytes": (SZ, [I32, I32]),
        "lk_latent_decode_attn_rope": (C.c_int, [CP, CP, P, C.c_int, P, P, C.c_int, I32, P, I32, P, C.c_float, P,
                                                 C.c_int, P, SZ, P]),
        "lk_latent_decode_rope_workspace_bytes": (SZ, [CP, CP, I32, I32]),
        "lk_lowrank_linear": (C.c_int, [WP, P, P, I32, P, P, C.c_int, P, P, P, SZ, P]),
        "lk_lowrank_workspace_bytes": (SZ, [WP, I32]),
        "lk_quantize_latent": (C.c_int, [P, I32, I32, C.c_int, I32, P, P, P]),
        "lk_quantize_rows_i8": (C.c_int, [P, C.c_int, I32, I32, P, P, P]),
        "lk_rmsnorm_quant_i8": (C.c_int, [P, C.c_int, I32, I32, C.c_float, P, P, P]),
        "lk_rmsnorm_hadamard_quant_i8": (C.c_int, [P, C.c_int, I32, I32, C.c_float, P, P, P]),
        "lk_swiglu_quant_i8": (C.c_int, [P, P, C.c_int, I32, I32, P, P, P]),
        "lk_device_status": (C.c_int, [I32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def check(status):
    """Raise LkError for a non-OK status, with the library's last error text."""
    if status != LK_OK:
        raise LkError(status, lib.lk_last_error().decode(errors="replace"))
