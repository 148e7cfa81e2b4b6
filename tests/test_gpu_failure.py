"""The expired-wait path of the decode kernel, made to happen on purpose.

A test hook (lk_debug_decode_attn_stall) runs the decode attention with its
copy producer stopping before one work item, as if that copy never came, and
the pipeline waits bounded by a few milliseconds.  The waits behind the
missing copy must expire; the kernel must still let the copies it started
land and return; lk_device_status() must then report
LK_ERR_DEVICE once, and the context must stay usable: the next ordinary call
gives the right answer and leaves its workspace counters at zero.  Nothing
here faults or hangs the GPU: the stall is a copy that is never issued, and
every wait in the kernel has a limit.
"""
import ctypes as C
import math

import numpy as np
import pytest
import torch

from tests.helpers import assert_close_rms, build_caches

pytestmark = pytest.mark.gpu


def _case(seed, kind="i8"):
    import rank_latent_kv_lk_b200 as lk
    ranks_k, ranks_v, H = [32, 16, 64, 8], [16, 64, 32, 8], 128
    if kind == "i4":
        ranks_k, ranks_v = [24, 16, 32, 8], [16, 32, 24, 8]
    lens = [1500, 700]
    B = len(lens)
    rng = np.random.default_rng(seed)
    lat_k = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_k] for b in range(B)]
    lat_v = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_v] for b in range(B)]
    _, _, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, kind, 32)
    ck = lk.LatentCache(B, ranks_k, 1504, kind, 32)
    cv = lk.LatentCache(B, ranks_v, 1504, kind, 32, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(seed)
    BK = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(torch.bfloat16).cuda()
    BV = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(torch.bfloat16).cuda()
    q = torch.randn(B, len(ranks_k), H, generator=g).to(torch.bfloat16).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return lk, ck, cv, BK, BV, q, seq, lens, H


@pytest.mark.parametrize("kind,stall_item", [("i8", 0), ("i8", 5), ("i4", 3)])
def test_stalled_copy_expires_reports_and_recovers(kind, stall_item):
    lk, ck, cv, BK, BV, q, seq, lens, H = _case(61, kind)
    from rank_latent_kv_lk_b200 import _lib
    ref = lk.latent_decode_attn(ck, cv, q, BK, BV, seq, max(lens), out_dtype=torch.float32).clone()
    torch.cuda.synchronize()
    lk.device_status()
    need = _lib.lib.lk_latent_decode_workspace_bytes(ck.desc(), cv.desc(), max(lens), 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.zeros_like(ref)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _lib.lib.lk_debug_decode_attn_stall(
        ck.desc(), cv.desc(), C.c_void_p(q.data_ptr()), _lib.LK_BF16, C.c_void_p(BK.data_ptr()),
        C.c_void_p(BV.data_ptr()), _lib.LK_BF16, H, C.c_void_p(seq.data_ptr()), max(lens), 1.0 / math.sqrt(H),
        C.c_void_p(out.data_ptr()), _lib.LK_F32, 0, C.c_void_p(ws.data_ptr()), ws.numel(), stall_item, 5000, stream)
    assert st == _lib.LK_OK, _lib.lib.lk_last_error()
    # the kernel returned (this synchronises) and reported the expired waits
    assert _lib.lib.lk_device_status(1) == _lib.LK_ERR_DEVICE
    assert b"bounded wait" in _lib.lib.lk_last_error()
    assert _lib.lib.lk_device_status(1) == _lib.LK_OK  # reported once, then cleared
    # the same workspace serves the next ordinary call: its counters are zero
    assert int(ws[:256].count_nonzero()) == 0
    out2 = torch.full_like(ref, float("nan"))
    st = _lib.lib.lk_latent_decode_attn(
        ck.desc(), cv.desc(), C.c_void_p(q.data_ptr()), _lib.LK_BF16, C.c_void_p(BK.data_ptr()),
        C.c_void_p(BV.data_ptr()), _lib.LK_BF16, H, C.c_void_p(seq.data_ptr()), max(lens), 1.0 / math.sqrt(H),
        C.c_void_p(out2.data_ptr()), _lib.LK_F32, 0, C.c_void_p(ws.data_ptr()), ws.numel(), stream)
    assert st == _lib.LK_OK
    torch.cuda.synchronize()
    lk.device_status()
    assert_close_rms(out2.cpu().numpy(), ref.cpu().numpy(), 1e-5, "after the expired call")


def test_stall_hook_rejects_bad_arguments():
    from rank_latent_kv_lk_b200 import _lib
    st = _lib.lib.lk_debug_decode_attn_stall(None, None, None, 0, None, None, 0, 128, None, 0, 0.1, None, 0, 0, None,
                                             0, -1, 5000, None)
    assert st == _lib.LK_ERR_INVALID_ARG
