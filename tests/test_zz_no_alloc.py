"""The allocation-free decode attention entry point against the workspace one.

Some callers cannot allocate device memory at all: no cudaMalloc, no scratch
buffer of their own -- for instance code that runs under an allocator which
forbids new device allocations, or a runtime that only hands over tensors it
already owns.  lk_latent_decode_attn_noalloc serves them: its split-K scratch
lives in a static device array inside the library.  Here it is called through
the C ABI and must match lk_latent_decode_attn (same inputs, caller workspace)
within the 1e-5 * RMS bound used for fp32 outputs, on two calls in a row --
the second call reuses the array exactly as the first one left it -- and on a
sequence of calls whose batch changes, with a call rejected for its size in
between.

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


def _case(seed, ranks_k=(16, 32, 8, 64), ranks_v=(32, 8, 64, 16), lens=(700, 33, 2049), cap=2064):
    import rank_latent_kv_lk_b200 as lk
    ranks_k, ranks_v, lens, H = list(ranks_k), list(ranks_v), list(lens), 128
    B = len(lens)
    rng = np.random.default_rng(seed)
    lat_k = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_k] for b in range(B)]
    lat_v = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_v] for b in range(B)]
    _, _, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, "i8", 32)
    ck = lk.LatentCache(B, ranks_k, cap, "i8", 32)
    cv = lk.LatentCache(B, ranks_v, cap, "i8", 32, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(seed)
    BK = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(torch.bfloat16).cuda()
    BV = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(torch.bfloat16).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return lk, ck, cv, BK, BV, seq, lens, H, g


def _noalloc_call(case, q, max_len, n_split, out):
    lk, ck, cv, BK, BV, seq, lens, H, g = case
    from rank_latent_kv_lk_b200 import _lib
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _lib.lib.lk_latent_decode_attn_noalloc(
        ck.desc(), cv.desc(), C.c_void_p(q.data_ptr()), _lib.LK_BF16, C.c_void_p(BK.data_ptr()),
        C.c_void_p(BV.data_ptr()), _lib.LK_BF16, H, C.c_void_p(seq.data_ptr()), int(max_len),
        1.0 / math.sqrt(H), C.c_void_p(out.data_ptr()), _lib.LK_F32, int(n_split), stream)


def _check_against_workspace_call(case, what):
    """One accepted no-alloc call, compared with lk_latent_decode_attn on the same q."""
    lk, ck, cv, BK, BV, seq, lens, H, g = case
    from rank_latent_kv_lk_b200 import _lib
    q = torch.randn(len(lens), len(ck.ranks), H, generator=g).to(torch.bfloat16).cuda()
    ref = lk.latent_decode_attn(ck, cv, q, BK, BV, seq, max(lens), out_dtype=torch.float32)
    out = torch.full_like(ref, float("nan"))
    st = _noalloc_call(case, q, max(lens), 0, out)
    assert st == _lib.LK_OK, _lib.lib.lk_last_error()
    torch.cuda.synchronize()
    lk.device_status()
    assert_close_rms(out.cpu().numpy(), ref.cpu().numpy(), 1e-5, what)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    case = _case(41)
    for call in range(2):
        _check_against_workspace_call(case, f"call {call}")


def test_noalloc_shape_changes_and_a_rejected_call_in_between():
    """The array keeps the last call's partials, which may lie where a call of
    another B * n_heads keeps its arrival counters.  A call of a new shape
    clears them; a call rejected for its size must change nothing, so that a
    retry of the same shape (what the error message suggests) still clears."""
    from rank_latent_kv_lk_b200 import _lib
    small = _case(43, ranks_k=[32] * 32, ranks_v=[32] * 32, lens=[1500], cap=1504)
    big = _case(44, ranks_k=[16, 32, 64, 48] * 8, ranks_v=[64, 8, 32, 16] * 8,
                lens=[300, 1200, 17, 640, 999, 1, 450, 800], cap=8192)
    _check_against_workspace_call(small, "B = 1 before the rejected call")
    lk, ck, cv, BK, BV, seq, lens, H, g = big
    q = torch.randn(len(lens), len(ck.ranks), H, generator=g).to(torch.bfloat16).cuda()
    out = torch.full((len(lens), len(ck.ranks), H), 7.0, dtype=torch.float32, device="cuda")
    # B * n_heads = 256 units cut into 64 pieces each over 8192 positions: far
    # more partials than the static array holds
    st = _noalloc_call(big, q, 8192, 64, out)
    assert st == _lib.LK_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool(torch.all(out == 7.0)), "a rejected call wrote its output"
    _check_against_workspace_call(big, "B = 8 after the rejected call")
    _check_against_workspace_call(small, "B = 1 after B = 8")
    _check_against_workspace_call(big, "B = 8 again")
    _check_against_workspace_call(big, "B = 8, same shape twice")


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
