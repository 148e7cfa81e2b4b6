"""CPU-only checks of the C ABI: the library builds, loads, exports every
declared symbol, and rejects bad arguments on the host before any launch.

Device pointers passed here are fake; every call is expected to fail host
validation before touching CUDA (a call that got through would report
LK_ERR_CUDA on a machine without a GPU, which the tests treat as a failure).
"""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__.build()
    from rank_latent_kv_lk_b200 import _lib
    return _lib


def declared_functions():
    with open(os.path.join(ROOT, "include", "lk.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lk_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L.lib, n), n


def test_version_and_status_strings(L):
    assert L.lib.lk_version() == 1
    for s in range(10):
        assert L.lib.lk_status_string(s)
    assert L.lib.lk_status_string(99) == b"unknown status"


FAKE = 0x7F0000000000  # 256-byte aligned fake device address


def cache(L, batch=1, heads=2, cap=64, kind=None, group=32, ranks=(16, 16), codes=FAKE, scales=FAKE + 0x100000):
    r = (C.c_int32 * len(ranks))(*ranks)
    d = L.LatentCacheDesc(batch, heads, cap, L.LK_I8 if kind is None else kind, group, r, codes, scales)
    d._keep = r
    return d


def decode(L, k, v, max_len=32, ws_bytes=1 << 20, ws=FAKE + 0x200000, H=64, q=FAKE + 0x300000, n_split=0,
           qdt=None, outdt=None):
    return L.lib.lk_latent_decode_attn(C.byref(k), C.byref(v), C.c_void_p(q), L.LK_BF16 if qdt is None else qdt,
                                       C.c_void_p(FAKE + 0x400000), C.c_void_p(FAKE + 0x500000), L.LK_BF16, H,
                                       C.c_void_p(FAKE + 0x600000), max_len, 0.125,
                                       C.c_void_p(FAKE + 0x700000), L.LK_F32 if outdt is None else outdt, n_split,
                                       C.c_void_p(ws), ws_bytes, None)


def test_decode_validation(L):
    k, v = cache(L), cache(L)
    assert decode(L, cache(L, heads=0), v) == L.LK_ERR_SHAPE
    assert decode(L, cache(L, cap=40), v) == L.LK_ERR_SHAPE                   # capacity % 16
    assert decode(L, cache(L, ranks=(16, 18)), v) == L.LK_ERR_SHAPE           # rank % 4
    assert decode(L, cache(L, ranks=(16, 128)), v) == L.LK_ERR_SHAPE          # rank > 64
    assert decode(L, cache(L, kind=L.LK_I4, ranks=(12, 16)), cache(L, kind=L.LK_I4)) == L.LK_ERR_SHAPE
    assert decode(L, cache(L, kind=L.LK_I4, group=12), cache(L, kind=L.LK_I4)) == L.LK_ERR_SHAPE
    assert decode(L, cache(L, kind=7), v) == L.LK_ERR_DTYPE
    assert decode(L, cache(L, codes=FAKE + 16), v) == L.LK_ERR_ALIGN
    assert decode(L, k, cache(L, batch=2)) == L.LK_ERR_SHAPE
    assert decode(L, k, cache(L, kind=L.LK_I4)) == L.LK_ERR_UNSUPPORTED
    assert decode(L, k, v, max_len=65) == L.LK_ERR_SHAPE                      # beyond capacity
    assert decode(L, k, v, H=0) == L.LK_ERR_SHAPE
    assert decode(L, k, v, H=60) == L.LK_ERR_SHAPE                           # not a multiple of 8
    assert decode(L, k, v, q=FAKE + 0x300008) == L.LK_ERR_ALIGN
    assert decode(L, k, v, H=300) == L.LK_ERR_SHAPE
    assert decode(L, k, v, q=0) == L.LK_ERR_INVALID_ARG
    assert decode(L, k, v, qdt=L.LK_I8) == L.LK_ERR_DTYPE
    assert decode(L, k, v, outdt=L.LK_I4) == L.LK_ERR_DTYPE
    assert decode(L, k, v, n_split=-1) == L.LK_ERR_SHAPE
    assert decode(L, k, v, ws_bytes=16) == L.LK_ERR_WORKSPACE
    assert decode(L, k, v, ws=FAKE + 0x200010) == L.LK_ERR_ALIGN
    assert L.lib.lk_last_error()


def test_decode_workspace_size_formula(L):
    k, v = cache(L), cache(L)
    # counters (1 * 2 heads * 4 B, rounded to 256) + two partial slots per CTA of
    # (2 + 16) floats rounded to 20; items = units * ceil(max_len / 224)
    n = L.lib.lk_latent_decode_workspace_bytes(C.byref(k), C.byref(v), 64, 0)
    assert n == 256 + 2 * 2 * 20 * 4            # 2 items -> at most 2 CTAs
    n = L.lib.lk_latent_decode_workspace_bytes(C.byref(k), C.byref(v), 1000, 3)
    assert n == 256 + 6 * 2 * 20 * 4            # 10 items, about 3 pieces per unit -> 6 CTAs
    n = L.lib.lk_latent_decode_workspace_bytes(C.byref(k), C.byref(v), 64 * 1024, 0)
    assert n == 256 + 586 * 2 * 20 * 4          # 586 items, automatic grid (at most 1024 CTAs)


def test_step_validates_attention_before_launching(L):
    k, v = cache(L), cache(L)
    hl = (C.c_int32 * 1)(0)
    st = L.lib.lk_latent_decode_step(C.byref(k), C.byref(v), C.c_void_p(FAKE + 0x800000), L.LK_BF16, None,
                                     C.c_void_p(FAKE + 0xA00000), L.LK_BF16, None, 512, C.c_void_p(FAKE + 0xB00000),
                                     hl, C.c_void_p(FAKE + 0x300000), L.LK_BF16, C.c_void_p(FAKE + 0x400000),
                                     C.c_void_p(FAKE + 0x500000), L.LK_BF16, 60, 0.125, C.c_void_p(FAKE + 0x700000),
                                     L.LK_F32, 0, C.c_void_p(FAKE + 0x900000), 1 << 24, C.c_void_p(FAKE + 0x200000),
                                     1 << 20, None)
    assert st == L.LK_ERR_SHAPE  # head_dim 60: rejected before the append is launched


def project(L, k, v, x=FAKE + 0x800000, xdt=None, E=512, n_new=1, host_len=(0,), ws_bytes=1 << 24,
            ws=FAKE + 0x900000, x_scale=None, a_scale=None):
    hl = (C.c_int32 * len(host_len))(*host_len)
    return L.lib.lk_latent_project_append(C.byref(k), C.byref(v), C.c_void_p(x), L.LK_F32 if xdt is None else xdt,
                                          x_scale, C.c_void_p(FAKE + 0xA00000), L.LK_F32 if xdt is None else xdt,
                                          a_scale, E, n_new, C.c_void_p(FAKE + 0xB00000), hl, C.c_void_p(ws),
                                          ws_bytes, None)


def test_project_validation(L):
    k, v = cache(L), cache(L)
    assert project(L, k, v, host_len=(60,), n_new=5) == L.LK_ERR_CAPACITY
    assert project(L, k, v, host_len=(-1,)) == L.LK_ERR_SHAPE
    assert project(L, k, v, E=510) == L.LK_ERR_ALIGN
    assert project(L, k, v, x=FAKE + 4) == L.LK_ERR_ALIGN
    assert project(L, k, v, xdt=L.LK_I8) == L.LK_ERR_INVALID_ARG            # int8 needs scales
    assert project(L, k, v, xdt=L.LK_F16) == L.LK_ERR_DTYPE
    assert project(L, k, v, n_new=0) == L.LK_ERR_SHAPE
    assert project(L, k, v, ws_bytes=8) == L.LK_ERR_WORKSPACE
    assert project(L, k, cache(L, batch=3), host_len=(0, 0, 0)) == L.LK_ERR_SHAPE


def lowrank(L, k_in=64, n_out=32, rank=16, n_dense=16, m=2, ws_bytes=1 << 24, tq=None):
    w = L.LowrankWeightDesc(k_in, n_out, rank, n_dense, *[C.c_void_p(FAKE + i * 0x10000) for i in range(8)])
    return L.lib.lk_lowrank_linear(C.byref(w), C.c_void_p(FAKE + 0xC00000), C.c_void_p(FAKE + 0xD00000), m,
                                   None, C.c_void_p(FAKE + 0xE00000), L.LK_BF16, tq, None,
                                   C.c_void_p(FAKE + 0xF00000), ws_bytes, None)


def test_lowrank_validation(L):
    assert lowrank(L, n_dense=8) == L.LK_ERR_ALIGN
    assert lowrank(L, rank=0) == L.LK_ERR_SHAPE          # low-rank channels without rank
    assert lowrank(L, n_dense=64, rank=16) == L.LK_ERR_SHAPE  # rank without channels
    assert lowrank(L, n_dense=80) == L.LK_ERR_SHAPE
    assert lowrank(L, m=-1) == L.LK_ERR_SHAPE
    assert lowrank(L, ws_bytes=0) == L.LK_ERR_WORKSPACE
    assert lowrank(L, tq=C.c_void_p(FAKE + 3)) == L.LK_ERR_ALIGN


def test_quantizer_validation(L):
    assert L.lib.lk_quantize_latent(None, 1, 65, L.LK_I8, 32, None, None, None) == L.LK_ERR_SHAPE
    assert L.lib.lk_quantize_latent(None, 1, 7, L.LK_I4, 32, None, None, None) == L.LK_ERR_SHAPE
    assert L.lib.lk_quantize_latent(None, 1, 8, L.LK_I8, 32, None, None, None) == L.LK_ERR_INVALID_ARG
    assert L.lib.lk_quantize_rows_i8(None, L.LK_F32, 1, 40000, None, None, None) == L.LK_ERR_SHAPE
    assert L.lib.lk_quantize_rows_i8(None, L.LK_I8, 1, 4, None, None, None) == L.LK_ERR_DTYPE
    assert L.lib.lk_rmsnorm_quant_i8(None, L.LK_F32, 1, 4, -1.0, None, None, None) == L.LK_ERR_INVALID_ARG
    assert L.lib.lk_rmsnorm_hadamard_quant_i8(None, L.LK_F32, 1, 48, 1e-5, None, None, None) == L.LK_ERR_SHAPE
    assert L.lib.lk_rmsnorm_hadamard_quant_i8(None, L.LK_F32, 1, 65536, 1e-5, None, None, None) == L.LK_ERR_SHAPE
    assert L.lib.lk_rmsnorm_hadamard_quant_i8(None, L.LK_F32, 1, 64, 1e-5, None, None, None) == L.LK_ERR_INVALID_ARG
    assert L.lib.lk_swiglu_quant_i8(C.c_void_p(FAKE), None, L.LK_F32, 1, 4, C.c_void_p(FAKE),
                                    C.c_void_p(FAKE), None) == L.LK_ERR_INVALID_ARG


def test_cache_bytes(L):
    k = cache(L, batch=3, heads=2, cap=64, ranks=(8, 24))
    cb, sb = C.c_size_t(), C.c_size_t()
    assert L.lib.lk_latent_cache_bytes(C.byref(k), C.byref(cb), C.byref(sb)) == L.LK_OK
    assert cb.value == 3 * 32 * 64 and sb.value == 3 * 2 * 64 * 4
    k4 = cache(L, batch=2, heads=2, cap=32, kind=L.LK_I4, group=16, ranks=(24, 64))
    assert L.lib.lk_latent_cache_bytes(C.byref(k4), C.byref(cb), C.byref(sb)) == L.LK_OK
    assert cb.value == 2 * (12 + 32) * 32 and sb.value == 2 * (2 + 4) * 32 * 2
    k.rotation = 1
    assert L.lib.lk_latent_cache_bytes(C.byref(k), C.byref(cb), C.byref(sb)) == L.LK_OK
    k.rotation = 2
    assert L.lib.lk_latent_cache_bytes(C.byref(k), C.byref(cb), C.byref(sb)) == L.LK_ERR_INVALID_ARG


def rope(L, k, v, max_len=32, ws_bytes=1 << 20, ws=FAKE + 0x200000, H=64, table=FAKE + 0xC00000, bdt=None):
    return L.lib.lk_latent_decode_attn_rope(C.byref(k), C.byref(v), C.c_void_p(FAKE + 0x300000), L.LK_BF16,
                                            C.c_void_p(FAKE + 0x400000), C.c_void_p(FAKE + 0x500000),
                                            L.LK_BF16 if bdt is None else bdt, H, C.c_void_p(FAKE + 0x600000),
                                            max_len, C.c_void_p(table), 0.125, C.c_void_p(FAKE + 0x700000),
                                            L.LK_F32, C.c_void_p(ws), ws_bytes, None)


def test_rope_validation(L):
    k, v = cache(L), cache(L)
    assert L.lib.lk_rope_table(7, 16, 10000.0, C.c_void_p(FAKE), None) == L.LK_ERR_SHAPE
    assert L.lib.lk_rope_table(64, -1, 10000.0, C.c_void_p(FAKE), None) == L.LK_ERR_SHAPE
    assert L.lib.lk_rope_table(64, 16, 1.0, C.c_void_p(FAKE), None) == L.LK_ERR_INVALID_ARG
    assert L.lib.lk_rope_table(64, 16, 10000.0, None, None) == L.LK_ERR_INVALID_ARG
    assert rope(L, k, v, H=48) == L.LK_ERR_SHAPE                              # not a multiple of 32
    assert rope(L, k, v, bdt=L.LK_F32) == L.LK_ERR_DTYPE                      # factors are bf16 operands
    assert rope(L, k, v, table=0) == L.LK_ERR_INVALID_ARG
    assert rope(L, k, v, table=FAKE + 8) == L.LK_ERR_ALIGN
    assert rope(L, k, v, max_len=65) == L.LK_ERR_SHAPE
    assert rope(L, k, v, ws_bytes=16) == L.LK_ERR_WORKSPACE
    assert rope(L, k, cache(L, kind=L.LK_I4)) == L.LK_ERR_UNSUPPORTED
    assert L.lib.lk_latent_decode_rope_workspace_bytes(C.byref(k), C.byref(v), 64, 32) > 256
    assert L.lib.lk_latent_decode_rope_workspace_bytes(C.byref(k), C.byref(v), 48, 32) == 0


def test_reconstruct_validation(L):
    k, v = cache(L), cache(L)

    def rec(bdt=None, H=64, max_len=32, bk=FAKE + 0x400000):
        return L.lib.lk_latent_reconstruct_kv(C.byref(k), C.byref(v), C.c_void_p(bk), C.c_void_p(FAKE + 0x500000),
                                              L.LK_BF16 if bdt is None else bdt, H, C.c_void_p(FAKE + 0x600000),
                                              max_len, C.c_void_p(FAKE + 0x700000), C.c_void_p(FAKE + 0x800000), None)
    assert rec(bdt=L.LK_F32) == L.LK_ERR_DTYPE
    assert rec(H=40) == L.LK_ERR_SHAPE                                       # not a multiple of 16
    assert rec(max_len=65) == L.LK_ERR_SHAPE
    assert rec(bk=FAKE + 0x400008) == L.LK_ERR_ALIGN


def test_ffn_outsplit_validation(L):
    w = L.OutsplitWeightDesc(FAKE, FAKE + 0x1000, FAKE + 0x2000, FAKE + 0x3000, FAKE + 0x4000, FAKE + 0x5000)

    def ffn(k_in=256, n_out=64, n_dense=16, rank=32, m=4, ws_bytes=1 << 24, wd=None):
        return L.lib.lk_ffn_gate_up_swiglu(C.byref(w if wd is None else wd), C.byref(w), k_in, n_out, n_dense, rank,
                                           C.c_void_p(FAKE + 0x6000), C.c_void_p(FAKE + 0x7000),
                                           C.c_void_p(FAKE + 0x8000), C.c_void_p(FAKE + 0x9000), m,
                                           C.c_void_p(FAKE + 0xA000), C.c_void_p(FAKE + 0x100000), ws_bytes, None)
    assert ffn(k_in=250) == L.LK_ERR_SHAPE
    assert ffn(rank=24) == L.LK_ERR_SHAPE
    assert ffn(n_dense=65) == L.LK_ERR_SHAPE
    assert ffn(n_dense=64, rank=32) == L.LK_ERR_SHAPE          # no low-rank channel but a rank
    assert ffn(n_dense=16, rank=0) == L.LK_ERR_SHAPE
    assert ffn(ws_bytes=16) == L.LK_ERR_WORKSPACE
    bad = L.OutsplitWeightDesc(FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert ffn(wd=bad) == L.LK_ERR_ALIGN
    assert L.lib.lk_ffn_gate_up_swiglu_workspace_bytes(512, 32) >= 2 * 32 * 512 * 4
