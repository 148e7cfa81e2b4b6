"""The allocation-free decode attention entry point against the workspace one.

Some callers cannot allocate device memory at all: no cudaMalloc, no scratch
buffer of their own -- for instance code that runs under an allocator which
forbids new device allocations, or a runtime that only hands over tensors it
already owns.  lk_latent_decode_attn_noalloc serves them: its split-K scratch
lives in a static device array inside the library.  Here it is called through
the C ABI and must match lk_latent_decode_attn (same inputs, caller workspace)
within the 1e-5 * RMS bound used for fp32 outputs, on two calls in a row --
the second call reuses the array exactly as the first one left it.

This file is collected last so that a stop-at-first-failure run has already
run every other test; it builds all of its own state.
"""
import ctypes as C
import math

import numpy as np
import pytest
import torch

from tests.helpers import assert_close_rms, build_caches

pytestmark = pytest.mark.gpu


def _case(seed):
    import rank_latent_kv_lk_b200 as lk
    ranks_k, ranks_v, H = [16, 32, 8, 64], [32, 8, 64, 16], 128
    lens = [700, 33, 2049]
    B = len(lens)
    rng = np.random.default_rng(seed)
    lat_k = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_k] for b in range(B)]
    lat_v = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_v] for b in range(B)]
    _, _, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, "i8", 32)
    cap = 2064
    ck = lk.LatentCache(B, ranks_k, cap, "i8", 32)
    cv = lk.LatentCache(B, ranks_v, cap, "i8", 32, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(seed)
    BK = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(torch.bfloat16).cuda()
    BV = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(torch.bfloat16).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return lk, ck, cv, BK, BV, seq, lens, H, g


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lk, ck, cv, BK, BV, seq, lens, H, g = _case(41)
    from rank_latent_kv_lk_b200 import _lib
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        q = torch.randn(len(lens), len(ck.ranks), H, generator=g).to(torch.bfloat16).cuda()
        ref = lk.latent_decode_attn(ck, cv, q, BK, BV, seq, max(lens), out_dtype=torch.float32)
        out = torch.full_like(ref, float("nan"))
        st = _lib.lib.lk_latent_decode_attn_noalloc(
            ck.desc(), cv.desc(), C.c_void_p(q.data_ptr()), _lib.LK_BF16, C.c_void_p(BK.data_ptr()),
            C.c_void_p(BV.data_ptr()), _lib.LK_BF16, H, C.c_void_p(seq.data_ptr()), max(lens),
            1.0 / math.sqrt(H), C.c_void_p(out.data_ptr()), _lib.LK_F32, 0, stream)
        assert st == _lib.LK_OK, _lib.lib.lk_last_error()
        torch.cuda.synchronize()
        lk.device_status()
        assert_close_rms(out.cpu().numpy(), ref.cpu().numpy(), 1e-5, f"call {call}")


def test_noalloc_rejects_requests_beyond_its_scratch():
    from rank_latent_kv_lk_b200 import _lib
    ranks = (C.c_int32 * 128)(*([64] * 128))
    # fake, never-touched device pointers: the request is rejected before any launch
    fake = 0x7F0000000000
    d = _lib.LatentCacheDesc(64, 128, 32768, _lib.LK_I8, 32, ranks, fake, fake + 0x100000)
    st = _lib.lib.lk_latent_decode_attn_noalloc(
        C.byref(d), C.byref(d), C.c_void_p(fake), _lib.LK_BF16, C.c_void_p(fake), C.c_void_p(fake),
        _lib.LK_BF16, 128, C.c_void_p(fake), 32768, 0.1, C.c_void_p(fake), _lib.LK_F32, 256, None)
    assert st == _lib.LK_ERR_WORKSPACE
    assert b"scratch" in _lib.lib.lk_last_error()
