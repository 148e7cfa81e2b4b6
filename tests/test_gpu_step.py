"""The decode step entry point (append + attention with the attention launch
overlapping the append) against the two calls made one after the other, on
identical caches: same appended codes and scales, same output bits."""
import math

import pytest
import torch

from rank_latent_kv_lk_b200 import synth
from rank_latent_kv_lk_b200.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _state(lk, w, ctx, device):
    rk, rv = synth.ranks(w)
    rk, rv = rk[0], rv[0]
    A, BK, BV = synth.factors(w, 0, rk, rv)
    cap = (ctx + 32 + 15) // 16 * 16
    ck = lk.LatentCache(w.batch, rk, cap, w.kind, w.group, device)
    cv = lk.LatentCache(w.batch, rv, cap, w.kind, w.group, device, role="v")
    seq = torch.zeros(w.batch, dtype=torch.int32, device=device)
    g = torch.Generator().manual_seed(5)
    x_ctx = torch.randn(w.batch * ctx, w.embed_dim, generator=g).to(A.dtype).to(device)
    lk.latent_project_append(ck, cv, x_ctx, A.to(device), seq, [0] * w.batch)
    return ck, cv, seq, A.to(device), BK.to(device), BV.to(device), rk, rv


@pytest.mark.parametrize("wl,ctx", [(2, 700), (1, 256)])
def test_step_matches_separate_calls(wl, ctx):
    import rank_latent_kv_lk_b200 as lk
    w = WORKLOADS[wl]
    dev = torch.device("cuda")
    a = _state(lk, w, ctx, dev)
    b = _state(lk, w, ctx, dev)
    g = torch.Generator().manual_seed(9)
    for step in range(3):
        x = torch.randn(w.batch, w.embed_dim, generator=g).to(a[3].dtype).to(dev)
        q = torch.randn(w.batch, w.n_heads, w.head_dim, generator=g).to(a[3].dtype).to(dev)
        lens = [ctx + step] * w.batch
        ck, cv, seq, A, BK, BV = a[:6]
        out1 = lk.latent_decode_step(ck, cv, x, A, seq, lens, q, BK, BV, out_dtype=torch.float32)
        ck2, cv2, seq2, A2, BK2, BV2 = b[:6]
        lk.latent_project_append(ck2, cv2, x, A2, seq2, lens)
        out2 = lk.latent_decode_attn(ck2, cv2, q, BK2, BV2, seq2, lens[0] + 1, out_dtype=torch.float32)
        torch.cuda.synchronize()
        lk.device_status()
        assert seq.tolist() == seq2.tolist() == [ctx + step + 1] * w.batch
        assert torch.equal(ck.codes, ck2.codes) and torch.equal(cv.codes, cv2.codes)
        assert torch.equal(ck.scales, ck2.scales) and torch.equal(cv.scales, cv2.scales)
        assert torch.equal(out1, out2), f"step {step}: outputs differ"
        assert torch.isfinite(out1).all() and float(out1.abs().max()) > 0
