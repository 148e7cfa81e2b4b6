"""The decode step entry point (append, then attention launched so that it
overlaps the append's tail) against the two calls made one after the other,
on identical caches: same appended codes and scales, same seq_len, and the
same output within the fp32 parity bound (1e-5 of the output RMS; the step
may split the attention over a different grid, which changes only the
rounding of the merge) -- for one and several rows, ragged lengths and
ranks, int4 caches and int8 (W8A8) inputs."""
import dataclasses
import math

import pytest
import torch

from rank_latent_kv_lk_b200 import synth
from rank_latent_kv_lk_b200.configs import WORKLOADS

pytestmark = pytest.mark.gpu


def _same_output(out1, out2):
    rms = float(out2.double().pow(2).mean().sqrt())
    return float((out1 - out2).abs().max()) <= 1e-5 * rms


def _state(lk, w, ctx, device, shorten, extra=32):
    rk, rv = synth.ranks(w)
    rk, rv = rk[0], rv[0]
    A, BK, BV = synth.factors(w, 0, rk, rv)
    cap = (ctx + extra + 15) // 16 * 16
    ck = lk.LatentCache(w.batch, rk, cap, w.kind, w.group, device)
    cv = lk.LatentCache(w.batch, rv, cap, w.kind, w.group, device, role="v")
    seq = torch.zeros(w.batch, dtype=torch.int32, device=device)
    g = torch.Generator().manual_seed(5)
    x_ctx = torch.randn(w.batch * ctx, w.embed_dim, generator=g).to(A.dtype).to(device)
    lk.latent_project_append(ck, cv, x_ctx, A.to(device), seq, [0] * w.batch)
    # ragged rows: row b keeps only its first ctx - shorten[b] tokens
    lens = [ctx - s for s in shorten]
    seq.copy_(torch.tensor(lens, dtype=torch.int32))
    return ck, cv, seq, A.to(device), BK.to(device), BV.to(device), lens


CASES = [
    # (workload, batch, context, per-row shortening)
    (2, 1, 700, [0]),                                   # bf16, one row
    (2, 1, 4096, [0]),                                  # full context: the step's grid differs
    (1, 1, 256, [0]),                                   # fp32 activations and factors
    (4, 8, 300, [0, 17, 5, 40, 1, 0, 33, 16]),          # ragged ranks and lengths, 8 rows
    (3, 4, 500, [3, 0, 11, 7]),                         # int4 groups of 24, 4 rows
    (3, 16, 260, [i % 5 for i in range(16)]),           # 16 rows (tensor-core projection)
]


@pytest.mark.parametrize("wl,batch,ctx,shorten", CASES)
def test_step_matches_separate_calls(wl, batch, ctx, shorten):
    import rank_latent_kv_lk_b200 as lk
    w = dataclasses.replace(WORKLOADS[wl], batch=batch)
    dev = torch.device("cuda")
    a = _state(lk, w, ctx, dev, shorten)
    b = _state(lk, w, ctx, dev, shorten)
    lens = list(a[6])
    g = torch.Generator().manual_seed(9)
    for step in range(3):
        x = torch.randn(w.batch, w.embed_dim, generator=g).to(a[3].dtype).to(dev)
        q = torch.randn(w.batch, w.n_heads, w.head_dim, generator=g).to(a[3].dtype).to(dev)
        ck, cv, seq, A, BK, BV = a[:6]
        out1 = lk.latent_decode_step(ck, cv, x, A, seq, lens, q, BK, BV, out_dtype=torch.float32)
        ck2, cv2, seq2, A2, BK2, BV2 = b[:6]
        lk.latent_project_append(ck2, cv2, x, A2, seq2, lens)
        out2 = lk.latent_decode_attn(ck2, cv2, q, BK2, BV2, seq2, max(lens) + 1, out_dtype=torch.float32)
        torch.cuda.synchronize()
        lk.device_status()
        lens = [n + 1 for n in lens]
        assert seq.tolist() == seq2.tolist() == lens
        assert torch.equal(ck.codes, ck2.codes) and torch.equal(cv.codes, cv2.codes)
        assert torch.equal(ck.scales, ck2.scales) and torch.equal(cv.scales, cv2.scales)
        assert _same_output(out1, out2), f"step {step}: outputs differ"
        assert torch.isfinite(out1).all() and float(out1.abs().max()) > 0


def test_step_w8a8_inputs_match_separate_calls():
    """int8 x and A with per-token / per-latent-dim scales (the W8A8 layer's
    projection), 4 rows: exact int32 sums, then the stated scaling."""
    import rank_latent_kv_lk_b200 as lk
    w = dataclasses.replace(WORKLOADS[5], batch=4)
    dev = torch.device("cuda")
    rk, rv = [32] * w.n_heads, [32] * w.n_heads
    g = torch.Generator().manual_seed(21)
    A_q, a_scale = synth.int8_weight(g, sum(rk) + sum(rv), w.embed_dim)
    _, BK, BV = synth.factors(dataclasses.replace(w, act="bf16"), 0, rk, rv)
    A_q, a_scale, BK, BV = A_q.to(dev), a_scale.to(dev), BK.to(dev), BV.to(dev)
    ctx = 333
    states = []
    for _ in range(2):
        ck = lk.LatentCache(w.batch, rk, 384, "i8", 32, dev)
        cv = lk.LatentCache(w.batch, rv, 384, "i8", 32, dev, role="v")
        seq = torch.zeros(w.batch, dtype=torch.int32, device=dev)
        gx = torch.Generator().manual_seed(22)
        xq = torch.randint(-127, 128, (w.batch * ctx, w.embed_dim), generator=gx, dtype=torch.int8).to(dev)
        xs = (torch.rand(w.batch * ctx, generator=gx) * 0.02 + 0.01).to(dev)
        lk.latent_project_append(ck, cv, xq, A_q, seq, [0] * w.batch, x_scale=xs, a_scale=a_scale)
        states.append((ck, cv, seq))
    lens = [ctx] * w.batch
    for step in range(2):
        xq = torch.randint(-127, 128, (w.batch, w.embed_dim), generator=g, dtype=torch.int8).to(dev)
        xs = (torch.rand(w.batch, generator=g) * 0.02 + 0.01).to(dev)
        q = torch.randn(w.batch, w.n_heads, w.head_dim, generator=g).to(torch.bfloat16).to(dev)
        ck, cv, seq = states[0]
        out1 = lk.latent_decode_step(ck, cv, xq, A_q, seq, lens, q, BK, BV, x_scale=xs, a_scale=a_scale,
                                     out_dtype=torch.float32)
        ck2, cv2, seq2 = states[1]
        lk.latent_project_append(ck2, cv2, xq, A_q, seq2, lens, x_scale=xs, a_scale=a_scale)
        out2 = lk.latent_decode_attn(ck2, cv2, q, BK, BV, seq2, max(lens) + 1, out_dtype=torch.float32)
        torch.cuda.synchronize()
        lk.device_status()
        lens = [n + 1 for n in lens]
        assert seq.tolist() == seq2.tolist() == lens
        assert torch.equal(ck.codes, ck2.codes) and torch.equal(cv.codes, cv2.codes)
        assert torch.equal(ck.scales, ck2.scales) and torch.equal(cv.scales, cv2.scales)
        assert _same_output(out1, out2)
        assert math.isfinite(float(out1.abs().max()))


def test_step_many_calls_leave_workspace_clean():
    """Fifty steps in a row on one pair of workspaces: every call must leave
    the arrival counters zero, so each later step is as exact as the first."""
    import rank_latent_kv_lk_b200 as lk
    w = dataclasses.replace(WORKLOADS[2], batch=2)
    dev = torch.device("cuda")
    a = _state(lk, w, 200, dev, [0, 9], extra=64)
    b = _state(lk, w, 200, dev, [0, 9], extra=64)
    lens = list(a[6])
    g = torch.Generator().manual_seed(31)
    for step in range(50):
        x = torch.randn(w.batch, w.embed_dim, generator=g).to(torch.bfloat16).to(dev)
        q = torch.randn(w.batch, w.n_heads, w.head_dim, generator=g).to(torch.bfloat16).to(dev)
        out1 = lk.latent_decode_step(a[0], a[1], x, a[3], a[2], lens, q, a[4], a[5], out_dtype=torch.float32)
        lk.latent_project_append(b[0], b[1], x, b[3], b[2], lens)
        out2 = lk.latent_decode_attn(b[0], b[1], q, b[4], b[5], b[2], max(lens) + 1, out_dtype=torch.float32)
        lens = [n + 1 for n in lens]
        if step % 10 == 9:
            torch.cuda.synchronize()
            lk.device_status()
            assert a[2].tolist() == b[2].tolist() == lens
            assert _same_output(out1, out2)
            assert torch.equal(a[0].codes, b[0].codes) and torch.equal(a[1].codes, b[1].codes)
    ws = lk.api.workspaces.get("project", 0, dev)
    assert int(ws[:256].count_nonzero()) == 0
