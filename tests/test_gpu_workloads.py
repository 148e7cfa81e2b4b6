"""The product entry points on the workloads' own seeded inputs, against the oracle.

Each test drives lk_latent_project_append (context prefill) and
lk_latent_decode_step (decode steps) with the inputs that bench.py times --
the image tokens (sigma 1.5) of the LLaVA-like workloads, the x20 outlier
channels of the int4 workload, the ragged per-(layer, head) ranks of the
LASER workload -- and compares:

  * appended codes and scales with the oracle's quantisation of its own fp32
    latents (float64 projection of the same x and A), by the band rule
    (a code may differ by one only at a rounding tie, tests/helpers.py);
  * decode outputs (bf16) with oracle.latent_attention (K and V materialised)
    on the device's own cache, read back, within 1e-2 * RMS(out) plus half a
    bf16 ulp of the value.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from rank_latent_kv_lk_b200 import synth
from rank_latent_kv_lk_b200.configs import WORKLOADS
from tests.helpers import assert_close_bf16, check_codes_band

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def _unit_codes(cache, b, h, T):
    rows, sc = cache.read_unit(b, h, T)
    r = cache.ranks[h]
    codes = rows.view(np.int8) if cache.kind == "i8" else O.unpack_i4(rows, r)
    return codes, sc


def _check_rows(cache, b, positions, v32_rows, off, flips):
    """Band-rule check of the codes at `positions` of row b against the oracle's
    fp32 latents v32_rows [len(positions), N_tot] (cache heads start at column off)."""
    T = max(positions) + 1
    for h, r in enumerate(cache.ranks):
        codes, sc = _unit_codes(cache, b, h, T)
        g = min(cache.group, r)
        flips[0] += check_codes_band(codes[positions], sc[positions], v32_rows[:, off:off + r], cache.kind, g)
        off += r
    return off


def _oracle_unit(q_bh, ck, cv, b, h, T, BKh, BVh, H):
    """Oracle attention of one (b, h) over the device's cache (read back)."""
    kind, gk, gv = ck.kind, min(ck.group, ck.ranks[h]), min(cv.group, cv.ranks[h])
    ckc, cks = _unit_codes(ck, b, h, T)
    cvc, cvs = _unit_codes(cv, b, h, T)
    if kind == "i8":
        kh, vh = O.dequantize_i8(ckc, cks), O.dequantize_i8(cvc, cvs)
    else:
        kh, vh = O.dequantize_i4(ckc, cks, gk), O.dequantize_i4(cvc, cvs, gv)
    return O.attention_materialized(q_bh, kh, vh, BKh, BVh, 1.0 / math.sqrt(H))


def _heads(F, ranks):
    off = np.concatenate([[0], np.cumsum(ranks)])
    return [F[off[i]:off[i + 1]] for i in range(len(ranks))]


def test_llava7b_b1_decode_steps_vs_oracle():
    """Workload 2 as bench.py runs it: 4096 context tokens (the first 576
    'image' tokens sigma 1.5) prefilled through the library, then 16 decode
    steps through lk_latent_decode_step with the seeded x and q."""
    lk = _lk()
    w = WORKLOADS[2]
    dev = torch.device("cuda")
    rk, rv = (r[0] for r in synth.ranks(w))
    A, BK, BV = synth.factors(w, 0, rk, rv)
    ck = lk.LatentCache(w.batch, rk, w.capacity, w.kind, w.group, dev)
    cv = lk.LatentCache(w.batch, rv, w.capacity, w.kind, w.group, dev, role="v")
    seq = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    x_ctx = synth.context_tokens(w, 0)
    lk.latent_project_append(ck, cv, x_ctx.reshape(-1, w.embed_dim).to(dev), A.to(dev), seq, [0])
    torch.cuda.synchronize()
    lk.device_status()
    A64 = synth.as_numpy(A).T.astype(np.float64)
    BKh = _heads(synth.as_numpy(BK).astype(np.float64), rk)
    BVh = _heads(synth.as_numpy(BV).astype(np.float64), rv)
    flips = [0]
    # every context position of the image range, then a stride through the text
    pos = list(range(0, 576, 3)) + list(range(576, w.context, 37)) + [w.context - 1]
    v_ctx = O.latent_project_float(synth.as_numpy(x_ctx[0, pos]), A64)
    off = _check_rows(ck, 0, pos, v_ctx, 0, flips)
    _check_rows(cv, 0, pos, v_ctx, off, flips)
    x_dec, q = synth.decode_tokens(w, 0), synth.queries(w, 0)
    A_d, BK_d, BV_d = A.to(dev), BK.to(dev), BV.to(dev)
    lens = [w.context]
    worst = 0.0
    for j in range(16):
        out = lk.latent_decode_step(ck, cv, x_dec[j].to(dev), A_d, seq, lens, q[j].to(dev), BK_d, BV_d)
        torch.cuda.synchronize()
        lk.device_status()
        lens = [lens[0] + 1]
        assert seq.tolist() == lens
        v_new = O.latent_project_float(synth.as_numpy(x_dec[j]), A64)
        off = _check_rows(ck, 0, [lens[0] - 1], v_new, 0, flips)
        _check_rows(cv, 0, [lens[0] - 1], v_new, off, flips)
        if j % 5 == 0 or j == 15:
            qn = synth.as_numpy(q[j]).astype(np.float64)
            want = np.stack([_oracle_unit(qn[0, h], ck, cv, 0, h, lens[0], BKh[h], BVh[h], w.head_dim)
                             for h in range(w.n_heads)])
            worst = max(worst, assert_close_bf16(out[0].float().cpu().numpy(), want, 1e-2, f"step {j}"))
    print(f"workload 2: {flips[0]} code flips at ties; worst output error {worst:.2e} of RMS")


def test_llava7b_int4_outliers_vs_oracle():
    """Workload 3: B = 16, 8192 context tokens with 5 % of x channels x20,
    int4 latents (one group of 24), through the library's prefill (the
    tensor-core projection) and two decode steps; sampled positions and units."""
    lk = _lk()
    w = WORKLOADS[3]
    dev = torch.device("cuda")
    rk, rv = (r[0] for r in synth.ranks(w))
    A, BK, BV = synth.factors(w, 0, rk, rv)
    ck = lk.LatentCache(w.batch, rk, w.capacity, w.kind, w.group, dev)
    cv = lk.LatentCache(w.batch, rv, w.capacity, w.kind, w.group, dev, role="v")
    seq = torch.zeros(w.batch, dtype=torch.int32, device=dev)
    x_ctx = synth.context_tokens(w, 0)
    lk.latent_project_append(ck, cv, x_ctx.reshape(-1, w.embed_dim).to(dev), A.to(dev), seq, [0] * w.batch)
    torch.cuda.synchronize()
    lk.device_status()
    A64 = synth.as_numpy(A).T.astype(np.float64)
    BKh = _heads(synth.as_numpy(BK).astype(np.float64), rk)
    BVh = _heads(synth.as_numpy(BV).astype(np.float64), rv)
    flips = [0]
    rng = np.random.default_rng(3)
    for b in range(w.batch):
        pos = sorted(set(rng.integers(0, 576, 4).tolist() + rng.integers(576, w.context, 8).tolist()))
        v = O.latent_project_float(synth.as_numpy(x_ctx[b, pos].cpu()), A64)
        off = _check_rows(ck, b, pos, v, 0, flips)
        _check_rows(cv, b, pos, v, off, flips)
    del x_ctx
    torch.cuda.empty_cache()
    x_dec, q = synth.decode_tokens(w, 0), synth.queries(w, 0)
    A_d, BK_d, BV_d = A.to(dev), BK.to(dev), BV.to(dev)
    lens = [w.context] * w.batch
    for j in range(2):
        out = lk.latent_decode_step(ck, cv, x_dec[j].to(dev), A_d, seq, lens, q[j].to(dev), BK_d, BV_d)
        torch.cuda.synchronize()
        lk.device_status()
        lens = [n + 1 for n in lens]
        v_new = O.latent_project_float(synth.as_numpy(x_dec[j]), A64)
        for b in range(w.batch):
            off = _check_rows(ck, b, [lens[b] - 1], v_new[b:b + 1], 0, flips)
            _check_rows(cv, b, [lens[b] - 1], v_new[b:b + 1], off, flips)
        qn = synth.as_numpy(q[j]).astype(np.float64)
        units = [(b, (5 * b + j) % w.n_heads) for b in range(w.batch)]
        got = out.float().cpu().numpy()
        want = np.stack([_oracle_unit(qn[b, h], ck, cv, b, h, lens[b], BKh[h], BVh[h], w.head_dim)
                         for b, h in units])
        assert_close_bf16(np.stack([got[b, h] for b, h in units]), want, 1e-2, f"step {j}")
    print(f"workload 3: {flips[0]} code flips at ties")


def test_laser_ragged_layers_vs_oracle():
    """Workload 4: three of the 32 layers (the first, the last and the one
    whose K and V ranks have the largest standard deviation), all 8 rows live with 16384 context
    tokens prefilled through the library, one decode step through
    lk_latent_decode_step.  Every row's new codes; sampled context positions;
    outputs of every row for the narrowest, the widest and one middle head."""
    lk = _lk()
    w = WORKLOADS[4]
    dev = torch.device("cuda")
    rks, rvs = synth.ranks(w)
    spread = [float(np.std(rks[l] + rvs[l])) for l in range(w.n_layers)]
    layers = sorted({0, w.n_layers - 1, int(np.argmax(spread))})
    flips = [0]
    rng = np.random.default_rng(4)
    for l in layers:
        rk, rv = rks[l], rvs[l]
        A, BK, BV = synth.factors(w, l, rk, rv)
        ck = lk.LatentCache(w.batch, rk, w.capacity, w.kind, w.group, dev)
        cv = lk.LatentCache(w.batch, rv, w.capacity, w.kind, w.group, dev, role="v")
        seq = torch.zeros(w.batch, dtype=torch.int32, device=dev)
        x_ctx = synth.context_tokens(w, l)
        A_d, BK_d, BV_d = A.to(dev), BK.to(dev), BV.to(dev)
        lk.latent_project_append(ck, cv, x_ctx.reshape(-1, w.embed_dim).to(dev), A_d, seq, [0] * w.batch)
        torch.cuda.synchronize()
        lk.device_status()
        A64 = synth.as_numpy(A).T.astype(np.float64)
        for b in range(w.batch):
            pos = sorted(set(rng.integers(0, w.context, 6).tolist()))
            v = O.latent_project_float(synth.as_numpy(x_ctx[b, pos].cpu()), A64)
            off = _check_rows(ck, b, pos, v, 0, flips)
            _check_rows(cv, b, pos, v, off, flips)
        del x_ctx
        torch.cuda.empty_cache()
        x, q = synth.decode_tokens(w, l)[0], synth.queries(w, l)[0]
        lens = [w.context] * w.batch
        out = lk.latent_decode_step(ck, cv, x.to(dev), A_d, seq, lens, q.to(dev), BK_d, BV_d)
        torch.cuda.synchronize()
        lk.device_status()
        lens = [n + 1 for n in lens]
        assert seq.tolist() == lens
        v_new = O.latent_project_float(synth.as_numpy(x), A64)
        for b in range(w.batch):
            off = _check_rows(ck, b, [lens[b] - 1], v_new[b:b + 1], 0, flips)
            _check_rows(cv, b, [lens[b] - 1], v_new[b:b + 1], off, flips)
        tot = [a + c for a, c in zip(rk, rv)]
        heads = sorted({int(np.argmin(tot)), int(np.argmax(tot)), len(tot) // 2})
        BKh = _heads(synth.as_numpy(BK).astype(np.float64), rk)
        BVh = _heads(synth.as_numpy(BV).astype(np.float64), rv)
        qn = synth.as_numpy(q).astype(np.float64)
        got = out.float().cpu().numpy()
        units = [(b, h) for b in range(w.batch) for h in heads]
        want = np.stack([_oracle_unit(qn[b, h], ck, cv, b, h, lens[b], BKh[h], BVh[h], w.head_dim)
                         for b, h in units])
        assert_close_bf16(np.stack([got[b, h] for b, h in units]), want, 1e-2,
                          f"layer {l} heads {heads} (ranks K {[rk[h] for h in heads]}, V {[rv[h] for h in heads]})")
        del ck, cv
        torch.cuda.empty_cache()
    print(f"workload 4 layers {layers}: {flips[0]} code flips at ties")
