"""Pins for the CPU oracle: each check compares it with something other than itself.

Hand-worked fixtures (tests/golden/), closed forms, exact rational arithmetic,
library routines that are not the ones the oracle calls (torch's attention,
RMSNorm, SiLU, bf16 cast), brute force with scalar loops on tiny inputs, and
invariants.  All CPU-only.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _nearest_f32(fr):
    """Correctly rounded float32 of an exact rational, by bracketing (ties to even)."""
    x = np.float32(float(fr))
    lo = np.nextafter(x, np.float32(-np.inf), dtype=np.float32)
    hi = np.nextafter(x, np.float32(np.inf), dtype=np.float32)
    cands = [lo, x, hi]
    errs = [abs(Fraction(float(c)) - fr) for c in cands]
    best = min(errs)
    winners = [c for c, e in zip(cands, errs) if e == best]
    if len(winners) == 1:
        return winners[0]
    return [c for c in winners if (np.float32(c).view(np.uint32) & 1) == 0][0]


# ---------------------------------------------------------------- quantisers

@pytest.mark.parametrize("case", _gold("quant_i8_worked.json")["cases"], ids=lambda c: c["name"])
def test_quant_i8_worked(case):
    if "v_ulps" in case:
        ulp = np.float32(2.0 ** -149)
        v = np.array(case["v_ulps"], np.float64) * float(ulp)
        v = v.astype(np.float32)
        want_scale = np.float32(case["scale_ulps"] * float(ulp))
    else:
        v = np.array(case["v"], np.float32)
        want_scale = np.float32(case["scale"])
    codes, scale = O.quantize_i8(v)
    assert codes.dtype == np.int8
    assert codes.tolist() == case["codes"]
    assert scale.view(np.uint32) == want_scale.view(np.uint32)


def test_quant_i8_scale_is_correctly_rounded_quotient():
    rng = np.random.default_rng(1)
    a = np.abs(rng.standard_normal(2000).astype(np.float32)) * np.float32(3.0)
    a = np.concatenate([a, np.float32(2.0) ** rng.integers(-140, 100, 200).astype(np.float32)])
    for ai in a:
        v = np.array([ai, -ai / 3], np.float32)
        _, s = O.quantize_i8(v)
        want = _nearest_f32(Fraction(float(ai)) / 127)
        assert s.view(np.uint32) == np.float32(want).view(np.uint32), ai


def test_quant_i8_codes_are_rne_of_exact_quotient():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal((300, 16)) * 2.0).astype(np.float32)
    codes, s = O.quantize_i8(v)
    for i in range(0, 300, 7):
        for j in range(16):
            ratio = _nearest_f32(Fraction(float(v[i, j])) / Fraction(float(s[i])))
            # round half to even on the float32 ratio, by hand
            fl = math.floor(float(ratio))
            frac = float(ratio) - fl
            if frac > 0.5 or (frac == 0.5 and fl % 2 == 1):
                fl += 1
            assert codes[i, j] == max(-127, min(127, fl))


def test_quant_i8_properties():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal((500, 32)) * rng.uniform(0.01, 100, (500, 1))).astype(np.float32)
    codes, s = O.quantize_i8(v)
    err = np.abs(v.astype(np.float64) - O.dequantize_i8(codes, s))
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 1e-6))
    assert np.all(np.max(np.abs(codes.astype(np.int32)), axis=1) == 127)
    c2, s2 = O.quantize_i8(-v)
    assert np.array_equal(c2, -codes) and np.array_equal(s2, s)
    # exact power-of-two rescaling leaves codes unchanged and scales the scale
    c3, s3 = O.quantize_i8(v * np.float32(8.0))
    assert np.array_equal(c3, codes) and np.array_equal(s3, s * np.float32(8.0))


@pytest.mark.parametrize("case", _gold("quant_i4_worked.json")["cases"], ids=lambda c: c["name"])
def test_quant_i4_worked(case):
    v = np.array(case["v"], np.float32)
    codes, scales = O.quantize_i4(v, case["group"])
    assert codes.tolist() == case["codes"]
    assert scales.astype(np.float64).tolist() == case["scales"]
    if "packed" in case:
        packed = O.pack_i4(codes)
        assert packed.tolist() == case["packed"]
        assert O.unpack_i4(packed, v.shape[-1]).tolist() == case["codes"]
    if "dequant" in case:
        deq = O.dequantize_i4(codes, scales, case["group"])
        assert deq.tolist() == [float(x) for x in case["dequant"]]


def test_quant_i4_properties():
    rng = np.random.default_rng(4)
    v = (rng.standard_normal((400, 24)) * rng.uniform(0.01, 50, (400, 1))).astype(np.float32)
    codes, sc = O.quantize_i4(v, 24)
    s = sc.astype(np.float64)[:, 0]
    assert codes.min() >= -7 and codes.max() <= 7
    err = np.abs(v - O.dequantize_i4(codes, sc, 24))
    # the fp16 scale carries a relative rounding error of at most 2^-11, which can
    # push the largest element's ratio to 7 +- 7*2^-11 (still one code of 7)
    assert np.all(err <= s[:, None] * (0.5 + 7 * 2.0 ** -11) + 1e-30)
    assert np.all(np.max(np.abs(codes.astype(np.int32)), axis=1) == 7)
    c2, s2 = O.quantize_i4(-v, 24)
    assert np.array_equal(c2, -codes) and np.array_equal(s2, sc)
    allc = np.arange(-8, 8, dtype=np.int8)
    grid = np.stack(np.meshgrid(allc, allc), -1).reshape(-1, 2)
    assert np.array_equal(O.unpack_i4(O.pack_i4(grid), 2), grid)


def test_quantize_latents_splits_ragged_heads():
    v = np.array([[127.0, 0.0, 0.0, 0.0, 254.0]], np.float32)
    (c0, s0), (c1, s1) = O.quantize_latents(v, [2, 3], "i8", 32)
    assert c0.tolist() == [[127, 0]] and s0.tolist() == [1.0]
    assert c1.tolist() == [[0, 0, 127]] and s1.tolist() == [2.0]


# ---------------------------------------------------------------- projection

def test_project_w8a8_worked():
    g = _gold("project_w8a8_tiny.json")
    v = O.latent_project_w8a8(np.array(g["x_q"], np.int8), np.array(g["x_scale"], np.float32),
                              np.array(g["A"], np.int8), np.array(g["a_scale"], np.float16))
    assert v.dtype == np.float32 and v.tolist() == g["v"]


def test_project_float_brute_force():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 5)).astype(np.float32)
    A = rng.standard_normal((5, 4)).astype(np.float32)
    v = O.latent_project_float(x, A)
    for m in range(3):
        for n in range(4):
            acc = sum(Fraction(float(x[m, e])) * Fraction(float(A[e, n])) for e in range(5))
            assert v[m, n] == _nearest_f32(acc)


# ---------------------------------------------------------------- attention

def test_attention_worked():
    g = _gold("attention_tiny.json")
    ck = O.dequantize_i8(np.array(g["codes_k"]), np.array(g["scales_k"], np.float32))
    cv = O.dequantize_i8(np.array(g["codes_v"]), np.array(g["scales_v"], np.float32))
    for fn in (O.attention_materialized, O.attention_absorbed):
        o = fn(np.array(g["q"]), ck, cv, np.array(g["B_K"]), np.array(g["B_V"]), g["softmax_scale"])
        np.testing.assert_allclose(o, g["o"], rtol=0, atol=1e-15)


def _rand_cache(rng, T, r, kind="i8"):
    v = (rng.standard_normal((T, r)) * 1.3).astype(np.float32)
    if kind == "i8":
        c, s = O.quantize_i8(v)
        return O.dequantize_i8(c, s)
    c, s = O.quantize_i4(v, min(32, r))
    return O.dequantize_i4(c, s, min(32, r))


def test_identity_factors_reproduce_dense_attention():
    rng = np.random.default_rng(6)
    H, T = 64, 77
    ck, cv = _rand_cache(rng, T, H), _rand_cache(rng, T, H)
    q = rng.standard_normal(H)
    eye = np.eye(H)
    o = O.attention_materialized(q, ck, cv, eye, eye, 1 / math.sqrt(H))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None, None], torch.tensor(ck)[None, None], torch.tensor(cv)[None, None])
    np.testing.assert_allclose(o, ref[0, 0, 0].numpy(), rtol=0, atol=1e-12)


def test_selection_factors_pad_with_zero_columns():
    # B = [I_r | 0]: K is the latent padded with zero columns; r != H so a
    # transposed factor cannot even be applied
    rng = np.random.default_rng(7)
    r, H, T = 16, 40, 33
    ck, cv = _rand_cache(rng, T, r), _rand_cache(rng, T, r)
    q = rng.standard_normal(H)
    sel = np.zeros((r, H))
    sel[:, :r] = np.eye(r)
    o = O.attention_materialized(q, ck, cv, sel, sel, 0.3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q[:r])[None, None, None], torch.tensor(ck)[None, None],
        torch.tensor(cv)[None, None], scale=0.3)[0, 0, 0].numpy()
    np.testing.assert_allclose(o[:r], ref, rtol=0, atol=1e-12)
    assert np.all(o[r:] == 0)


def test_uniform_scores_give_mean_of_v():
    rng = np.random.default_rng(8)
    T, rk, rv, H = 50, 8, 12, 20
    ck, cv = _rand_cache(rng, T, rk), _rand_cache(rng, T, rv)
    BK, BV = rng.standard_normal((rk, H)), rng.standard_normal((rv, H))
    o = O.attention_materialized(np.zeros(H), ck, cv, BK, BV, 0.1)
    mean_latent = np.mean(cv, axis=0)          # closed form: uniform weights 1/T
    np.testing.assert_allclose(o, mean_latent @ BV, rtol=1e-12, atol=1e-12)


def test_dominant_score_selects_one_token():
    rng = np.random.default_rng(9)
    T, r, H = 40, 8, 16
    ck = np.zeros((T, r))
    ck[17, 0] = 1.0
    cv = _rand_cache(rng, T, r)
    BK = np.zeros((r, H))
    BK[0, 0] = 1.0
    BV = rng.standard_normal((r, H))
    q = np.zeros(H)
    q[0] = 1e3                                  # token 17 scores 1e3, all others 0
    o = O.attention_materialized(q, ck, cv, BK, BV, 1.0)
    np.testing.assert_allclose(o, cv[17] @ BV, rtol=1e-12, atol=1e-12)


def test_single_token_returns_its_value():
    rng = np.random.default_rng(10)
    ck, cv = _rand_cache(rng, 1, 8), _rand_cache(rng, 1, 8)
    BK, BV = rng.standard_normal((8, 12)), rng.standard_normal((8, 12))
    o = O.attention_materialized(rng.standard_normal(12), ck, cv, BK, BV, 0.5)
    np.testing.assert_allclose(o, cv[0] @ BV, rtol=1e-13, atol=1e-13)


def test_two_tokens_closed_form():
    rng = np.random.default_rng(11)
    ck, cv = rng.standard_normal((2, 3)), rng.standard_normal((2, 3))
    BK, BV = rng.standard_normal((3, 4)), rng.standard_normal((3, 4))
    q = rng.standard_normal(4)
    o = O.attention_materialized(q, ck, cv, BK, BV, 0.7)
    s = [0.7 * sum(sum(ck[t, i] * BK[i, d] for i in range(3)) * q[d] for d in range(4)) for t in range(2)]
    p1 = 1.0 / (1.0 + math.exp(s[0] - s[1]))   # logistic of the score gap
    v = [[sum(cv[t, i] * BV[i, d] for i in range(3)) for d in range(4)] for t in range(2)]
    want = [(1 - p1) * v[0][d] + p1 * v[1][d] for d in range(4)]
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-12)


def test_absorbed_equals_materialized_and_permutation_invariant():
    rng = np.random.default_rng(12)
    T, rk, rv, H = 129, 24, 40, 64
    ck, cv = _rand_cache(rng, T, rk, "i4"), _rand_cache(rng, T, rv)
    BK, BV = rng.standard_normal((rk, H)) / 5, rng.standard_normal((rv, H)) / 7
    q = rng.standard_normal(H)
    o1 = O.attention_materialized(q, ck, cv, BK, BV, 1 / 8)
    o2 = O.attention_absorbed(q, ck, cv, BK, BV, 1 / 8)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    perm = rng.permutation(T)
    o3 = O.attention_materialized(q, ck[perm], cv[perm], BK, BV, 1 / 8)
    np.testing.assert_allclose(o1, o3, rtol=1e-12, atol=1e-12)


def test_latent_attention_over_cache_brute_force():
    rng = np.random.default_rng(13)
    Bsz, ranks_k, ranks_v, H = 2, [2, 3], [3, 1], 3
    ck = O.LatentCache(Bsz, ranks_k, "i8", 32)
    cv = O.LatentCache(Bsz, ranks_v, "i4", 32)
    lens = [3, 2]
    for b in range(Bsz):
        vk = rng.standard_normal((lens[b], sum(ranks_k))).astype(np.float32)
        vv = rng.standard_normal((lens[b], sum(ranks_v))).astype(np.float32)
        ck.append(b, O.quantize_latents(vk, ranks_k, "i8", 32))
        cv.append(b, O.quantize_latents(vv, ranks_v, "i4", 32))
    BK = [rng.standard_normal((r, H)) for r in ranks_k]
    BV = [rng.standard_normal((r, H)) for r in ranks_v]
    q = rng.standard_normal((Bsz, 2, H))
    o = O.latent_attention(q, ck, cv, BK, BV, 0.6)
    for b in range(Bsz):
        for h in range(2):
            kc, ks = ck.codes[b][h], ck.scales[b][h]
            vc, vs = cv.codes[b][h], cv.scales[b][h]
            s = []
            for t in range(lens[b]):
                acc = 0.0
                for d in range(H):
                    kd = sum(float(kc[t, i]) * float(ks[t]) * BK[h][i, d] for i in range(ranks_k[h]))
                    acc += kd * q[b, h, d]
                s.append(0.6 * acc)
            z = sum(math.exp(si) for si in s)
            for d in range(H):
                want = 0.0
                for t in range(lens[b]):
                    vd = sum(float(vc[t, i]) * float(vs[t, 0]) * BV[h][i, d] for i in range(ranks_v[h]))
                    want += math.exp(s[t]) / z * vd
                assert abs(o[b, h, d] - want) <= 1e-12 * max(1.0, abs(want))


# ---------------------------------------------------------------- hybrid linear

def test_hybrid_worked():
    g = _gold("hybrid_tiny.json")
    y, t_q, s_t = O.linear_w8a8_hybrid(
        np.array(g["x_q"], np.int8), np.array(g["x_scale"], np.float32),
        np.array(g["dense_idx"]), np.array(g["lr_idx"]),
        np.array(g["W_D"], np.int8), np.array(g["s_D"], np.float16),
        np.array(g["U"], np.int8), np.array(g["s_U"], np.float16),
        np.array(g["V"], np.int8), np.array(g["s_V"], np.float16))
    assert t_q.tolist() == g["t_q"]
    np.testing.assert_allclose(y[0], g["y"], rtol=1e-6)


def _brute_int_matmul(a, b):
    M, K = a.shape
    N = b.shape[1]
    return np.array([[sum(int(a[m, k]) * int(b[k, n]) for k in range(K)) for n in range(N)]
                     for m in range(M)], dtype=np.int64)


def test_hybrid_all_dense_is_dense_gemm():
    rng = np.random.default_rng(14)
    M, K, N = 3, 9, 5
    x = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W = rng.integers(-127, 128, (K, N)).astype(np.int8)
    sx = rng.uniform(0.01, 0.1, M).astype(np.float32)
    sW = rng.uniform(0.001, 0.01, N).astype(np.float16)
    y, _, _ = O.linear_w8a8_hybrid(x, sx, np.arange(K), np.zeros(0, int), W, sW, None, None, None, None)
    acc = _brute_int_matmul(x, W)
    want = acc * sx.astype(np.float64)[:, None] * sW.astype(np.float64)[None, :]
    np.testing.assert_allclose(y, want, rtol=1e-15, atol=0)


def test_hybrid_no_dense_is_pure_low_rank():
    rng = np.random.default_rng(15)
    M, K, N, R = 2, 7, 4, 3
    x = rng.integers(-127, 128, (M, K)).astype(np.int8)
    U = rng.integers(-127, 128, (K, R)).astype(np.int8)
    V = rng.integers(-127, 128, (R, N)).astype(np.int8)
    sx = rng.uniform(0.01, 0.1, M).astype(np.float32)
    sU = rng.uniform(0.001, 0.01, R).astype(np.float16)
    sV = rng.uniform(0.001, 0.01, N).astype(np.float16)
    res = rng.standard_normal((M, N))
    y, t_q, s_t = O.linear_w8a8_hybrid(x, sx, np.zeros(0, int), np.arange(K), None, None,
                                      U, sU, V, sV, residual=res)
    accU = _brute_int_matmul(x, U)
    t = np.zeros((M, R), np.float32)
    for m in range(M):
        for k in range(R):
            t[m, k] = np.float32(np.float32(np.float32(accU[m, k]) * sx[m]) * np.float32(sU[k]))
    tq_want, st_want = O.quantize_i8(t)            # pinned separately above
    assert np.array_equal(t_q, tq_want) and np.array_equal(s_t, st_want)
    accV = _brute_int_matmul(t_q, V)
    want = accV * s_t.astype(np.float64)[:, None] * sV.astype(np.float64)[None, :] + res
    np.testing.assert_allclose(y, want, rtol=1e-14, atol=1e-14)


def test_hybrid_split_equals_sum_of_branches():
    # splitting the channels between the branches is a partition of one sum
    rng = np.random.default_rng(16)
    M, K, N = 2, 10, 6
    x = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W = rng.integers(-127, 128, (K, N)).astype(np.int8)
    sx = np.ones(M, np.float32)
    sW = np.ones(N, np.float16)
    D = np.array([0, 3, 4, 8])
    notD = np.array([1, 2, 5, 6, 7, 9])
    # low-rank branch with U = identity-like and V = W rows: t = x[:, notD] exactly,
    # requantised; choose rows so the absmax is 127 and the requant is exact
    x[:, notD[0]] = 127
    U = np.eye(len(notD), dtype=np.int8)
    V = W[notD]
    y, t_q, s_t = O.linear_w8a8_hybrid(x, sx, D, notD, W[D], sW, U, np.ones(len(notD), np.float16),
                                       V, np.ones(N, np.float16))
    assert np.array_equal(t_q, x[:, notD]) and np.all(s_t == 1.0)
    np.testing.assert_array_equal(y, _brute_int_matmul(x, W).astype(np.float64))


# ---------------------------------------------------------------- elementwise, norm, bf16

def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(17)
    x = rng.standard_normal((4, 33)) * 3
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (33,), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, 1e-5), ref, rtol=1e-14, atol=1e-14)


def test_swiglu_matches_torch_silu():
    rng = np.random.default_rng(18)
    g, u = rng.standard_normal(1000) * 6, rng.standard_normal(1000)
    ref = (torch.nn.functional.silu(torch.tensor(g)) * torch.tensor(u)).numpy()
    np.testing.assert_allclose(O.swiglu(g, u), ref, rtol=1e-14, atol=1e-15)
    assert O.swiglu(0.0, 5.0) == 0.0


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(19)
    x = np.concatenate([rng.standard_normal(5000).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1e-40, 3.4e38, -1.5], np.float32)])
    ref = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x), ref)


# ---------------------------------------------------------------- per-head SVD

@pytest.mark.parametrize("r", [1, 4, 9])
def test_per_head_svd_eckart_young(r):
    rng = np.random.default_rng(20)
    E, H = 48, 16
    Q1, _ = np.linalg.qr(rng.standard_normal((E, H)))
    Q2, _ = np.linalg.qr(rng.standard_normal((H, H)))
    sig = 2.0 ** (-np.arange(H) / 4)
    W = Q1 @ np.diag(sig) @ Q2.T
    A, B = O.per_head_svd(W, r)
    assert A.shape == (E, r) and B.shape == (r, H)
    err = W - A @ B
    fro2 = float(np.sum(sig[r:] ** 2))
    np.testing.assert_allclose(np.sum(err ** 2), fro2, rtol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(err, 2), sig[r], rtol=1e-10)


# ---------------------------------------------------------------- decoder layer

def test_decoder_layer_zero_branches_is_identity():
    """W_O = 0 and a zero down projection leave only the two residual adds."""
    rng = np.random.default_rng(21)
    Bsz, E, n_h, H, I = 2, 16, 2, 8, 12
    rk, rv = [4, 4], [4, 4]
    x = O.round_bf16(rng.standard_normal((Bsz, E)))

    def hyb(k_in, n, zero=False):
        D = np.sort(rng.choice(k_in, k_in // 4, replace=False))
        notD = np.setdiff1d(np.arange(k_in), D)
        R = 3
        w = lambda *s: (np.zeros(s, np.int8) if zero else rng.integers(-127, 128, s).astype(np.int8))
        return dict(dense_idx=D, lr_idx=notD, W_D=w(len(D), n), s_D=np.full(n, 0.01, np.float16),
                    U=w(len(notD), R), s_U=np.full(R, 0.01, np.float16), V=w(R, n),
                    s_V=np.full(n, 0.01, np.float16))

    layer = dict(
        n_heads=n_h, head_dim=H, ranks_k=rk, ranks_v=rv,
        W_Q=rng.integers(-127, 128, (E, n_h * H)).astype(np.int8), s_Q=np.full(n_h * H, 0.01, np.float16),
        W_O=np.zeros((n_h * H, E), np.int8), s_O=np.full(E, 0.01, np.float16),
        A=rng.integers(-127, 128, (E, 16)).astype(np.int8), s_A=np.full(16, 0.01, np.float16),
        B_K=[rng.standard_normal((4, H)) for _ in range(n_h)],
        B_V=[rng.standard_normal((4, H)) for _ in range(n_h)],
        gate=hyb(E, I), up=hyb(E, I), down=hyb(I, E, zero=True))
    ck, cv = O.LatentCache(Bsz, rk, "i8", 32), O.LatentCache(Bsz, rv, "i8", 32)
    out, inter = O.decoder_layer_w8a8(x, layer, ck, cv)
    np.testing.assert_array_equal(out, x)
    assert ck.length(0) == 1 and cv.length(1) == 1
    assert np.all(np.abs(inter["attn"]) > 0)


def test_decoder_layer_tiny_worked():
    """A whole layer step on a hand-worked example (tests/golden/decoder_layer_tiny.json).

    E = 4, one head with H = 2 and r_K = r_V = 1, one cached token, a 2-channel
    hybrid FFN.  Every stored intermediate is compared exactly (int8 codes,
    float32 scales, bf16 tensors); the float64 layer output to 1e-12 relative.
    The values fix which tensor feeds which stage: SwiGLU(gate, up) and not
    (up, gate), the FFN fed RMSNorm(x2) and not h1, the attention output
    stored as bf16 before it is quantised, both residuals."""
    gj = _gold("decoder_layer_tiny.json")
    inp, exp = gj["inputs"], gj["expected"]
    f16 = lambda a: np.asarray(a, np.float16)
    i8 = lambda a: np.asarray(a, np.int8)

    def hyb(w):
        return dict(dense_idx=np.asarray(w["dense_idx"]), lr_idx=np.asarray(w["lr_idx"]), W_D=i8(w["W_D"]),
                    s_D=f16(w["s_D"]), U=i8(w["U"]), s_U=f16(w["s_U"]), V=i8(w["V"]), s_V=f16(w["s_V"]))

    layer = dict(n_heads=1, head_dim=2, ranks_k=[1], ranks_v=[1],
                 W_Q=i8(inp["W_Q"]), s_Q=f16(inp["s_Q"]), W_O=i8(inp["W_O"]), s_O=f16(inp["s_O"]),
                 A=i8(inp["A"]), s_A=f16(inp["s_A"]),
                 B_K=[np.asarray(inp["B_K"], np.float64)], B_V=[np.asarray(inp["B_V"], np.float64)],
                 gate=hyb(inp["gate"]), up=hyb(inp["up"]), down=hyb(inp["down"]))
    ck, cv = O.LatentCache(1, [1], "i8", 32), O.LatentCache(1, [1], "i8", 32)
    tok = inp["cached_token"]
    ck.append(0, [(i8([[tok["k_code"]]]), np.asarray([tok["k_scale"]], np.float32))])
    cv.append(0, [(i8([[tok["v_code"]]]), np.asarray([tok["v_scale"]], np.float32))])
    out, inter = O.decoder_layer_w8a8(np.asarray(inp["x"], np.float64), layer, ck, cv, eps=0.0)

    hx = lambda a: np.vectorize(float.fromhex)(np.asarray(a, dtype=object)).astype(np.float64)
    for key in ("xq", "aq", "hq", "mq"):
        np.testing.assert_array_equal(np.asarray(inter[key], np.int64), np.asarray(exp[key], np.int64), err_msg=key)
    for key in ("sx", "sa", "sh", "sm"):
        got = np.asarray(inter[key], np.float32)
        np.testing.assert_array_equal(got.view(np.uint32), hx(exp[key]).astype(np.float32).view(np.uint32),
                                      err_msg=key)
    np.testing.assert_array_equal(np.asarray(inter["q"], np.float64), np.asarray(exp["q"], np.float64))
    for key in ("latent", "attn", "x2", "gate", "up"):
        np.testing.assert_array_equal(np.asarray(inter[key], np.float64), hx(exp[key]), err_msg=key)
    np.testing.assert_allclose(out, hx(exp["out"]), rtol=1e-12, atol=0)
    # the new token was appended behind the cached one with the quantiser's codes and scales
    assert ck.length(0) == 2 and cv.length(0) == 2
    for cache, (code, scale) in ((ck, exp["k_new"]), (cv, exp["v_new"])):
        assert int(cache.codes[0][0][1, 0]) == code
        assert np.float32(cache.scales[0][0][1]).view(np.uint32) == np.float32(float.fromhex(scale)).view(np.uint32)


# ---------------------------------------------------------------- rotations (S1, S2)

@pytest.mark.parametrize("n", [1, 2, 8, 64, 4096])
def test_hadamard_closed_form_and_orthogonal(n):
    """Sylvester-Hadamard entries are (-1)^popcount(i & j) / sqrt(n); the
    matrix is symmetric and orthogonal."""
    h = O.hadamard(n)
    if n <= 64:
        i = np.arange(n)[:, None]
        j = np.arange(n)[None, :]
        parity = np.vectorize(lambda a: bin(int(a)).count("1") & 1)(i & j)
        np.testing.assert_array_equal(h * math.sqrt(n), np.where(parity, -1.0, 1.0))
    np.testing.assert_allclose(h @ h.T, np.eye(n), atol=1e-12)
    np.testing.assert_array_equal(h, h.T)


@pytest.mark.parametrize("r,block", [(8, 8), (16, 16), (24, 8), (32, 32), (48, 16), (64, 64), (12, 4), (4, 4)])
def test_latent_rotation_blocks(r, block):
    s2 = O.latent_rotation(r)
    np.testing.assert_allclose(s2 @ s2.T, np.eye(r), atol=1e-12)
    for b0 in range(0, r, block):
        np.testing.assert_allclose(s2[b0:b0 + block, b0:b0 + block], O.hadamard(block))
        mask = np.ones(r, bool)
        mask[b0:b0 + block] = False
        assert np.all(s2[b0:b0 + block][:, mask] == 0)


def test_rotations_leave_attention_unchanged():
    """With the cache rotated (C S2) and the factor counter-rotated (S2^T B),
    materialised attention is the same (no quantisation in between)."""
    rng = np.random.default_rng(9)
    T, r, H = 37, 24, 16
    C, Cv = rng.standard_normal((T, r)), rng.standard_normal((T, r))
    BK, BV = rng.standard_normal((r, H)), rng.standard_normal((r, H))
    q = rng.standard_normal(H)
    s2 = O.latent_rotation(r)
    a = O.attention_materialized(q, C, Cv, BK, BV, 0.3)
    b = O.attention_materialized(q, C @ s2, Cv @ s2, s2.T @ BK, s2.T @ BV, 0.3)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    x = rng.standard_normal((3, 64))
    A = rng.standard_normal((64, 24))
    h = O.hadamard(64)
    np.testing.assert_allclose((x @ h) @ (h.T @ A), x @ A, atol=1e-12)


def test_rotate_latents_and_rmsnorm_hadamard_brute_force():
    rng = np.random.default_rng(10)
    ranks = [24, 8, 16]
    v = rng.standard_normal((2, sum(ranks))).astype(np.float32)
    got = O.rotate_latents(v, ranks)
    off = 0
    for r in ranks:
        n = r & -r if (r & -r) <= 64 else 64
        for row in range(2):
            for d in range(r):
                blk = (d // n) * n
                acc = sum(float(v[row, off + blk + i]) * (-1) ** bin(i & (d - blk)).count("1") for i in range(n))
                assert got[row, off + d] == np.float32(acc / math.sqrt(n))
        off += r
    x = rng.standard_normal((2, 8))
    y = O.rmsnorm_hadamard(x, 1e-5)
    xn = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-5)
    for row in range(2):
        for j in range(8):
            want = sum(xn[row, i] * (-1) ** bin(i & j).count("1") for i in range(8)) / math.sqrt(8)
            assert abs(y[row, j] - want) < 1e-12


# ---------------------------------------------------------------- rotary positions (extension)

def test_rope_unit_vectors_closed_form():
    """H = 8, base 10000: theta_i = 10^-i.  e_i at position p turns into
    cos(p theta_i) e_i + sin(p theta_i) e_{i+4}; e_{i+4} into
    cos(p theta_i) e_{i+4} - sin(p theta_i) e_i."""
    H, p = 8, 3
    for i in range(4):
        th = 10.0 ** (-i)
        e = np.zeros((1, H))
        e[0, i] = 1.0
        want = np.zeros(H)
        want[i], want[i + 4] = math.cos(p * th), math.sin(p * th)
        np.testing.assert_allclose(O.rope(e, [p])[0], want, atol=1e-15)
        e = np.zeros((1, H))
        e[0, i + 4] = 1.0
        want = np.zeros(H)
        want[i + 4], want[i] = math.cos(p * th), -math.sin(p * th)
        np.testing.assert_allclose(O.rope(e, [p])[0], want, atol=1e-15)
    # position 0 is the identity
    x = np.random.default_rng(1).standard_normal((3, 16))
    np.testing.assert_array_equal(O.rope(x, [0, 0, 0]), x)


def test_rope_scores_depend_on_offset_only():
    """<R_m q, R_n k> = <q, R_{n-m} k>: block rotation matrices built
    explicitly (2 x 2 per frequency pair), positions shifted together leave
    every score unchanged, and the rotation keeps norms."""
    rng = np.random.default_rng(2)
    H = 16
    q, k = rng.standard_normal(H), rng.standard_normal(H)

    def rot(pos):
        R = np.zeros((H, H))
        for i in range(H // 2):
            a = pos * 10000.0 ** (-2.0 * i / H)
            R[i, i], R[i, i + H // 2] = math.cos(a), -math.sin(a)
            R[i + H // 2, i], R[i + H // 2, i + H // 2] = math.sin(a), math.cos(a)
        return R

    for m, n in ((0, 5), (7, 3), (1000, 16383)):
        s = O.rope(q[None], [m])[0] @ O.rope(k[None], [n])[0]
        assert abs(s - q @ (rot(n - m) @ k)) < 1e-9 * (1 + abs(s))
        np.testing.assert_allclose(O.rope(k[None], [n])[0], rot(n) @ k, atol=1e-12)
        assert abs(np.linalg.norm(O.rope(k[None], [n])[0]) - np.linalg.norm(k)) < 1e-12


def test_attention_rope_brute_force_and_shift_invariance():
    rng = np.random.default_rng(3)
    T, r, H = 5, 4, 8
    Ck, Cv = rng.standard_normal((T, r)), rng.standard_normal((T, r))
    BK, BV = rng.standard_normal((r, H)), rng.standard_normal((r, H))
    q = rng.standard_normal(H)
    got = O.attention_rope(q, Ck, Cv, BK, BV, 0.4, q_pos=T - 1)
    # brute force: explicit per-pair rotations, scores, softmax, weighted V rows
    scores = []
    for t in range(T):
        kt = Ck[t] @ BK
        acc = 0.0
        for i in range(H // 2):
            th = 10000.0 ** (-2.0 * i / H)
            ck, sk = math.cos(t * th), math.sin(t * th)
            cq, sq = math.cos((T - 1) * th), math.sin((T - 1) * th)
            k1, k2 = kt[i] * ck - kt[i + 4] * sk, kt[i + 4] * ck + kt[i] * sk
            q1, q2 = q[i] * cq - q[i + 4] * sq, q[i + 4] * cq + q[i] * sq
            acc += k1 * q1 + k2 * q2
        scores.append(0.4 * acc)
    w = [math.exp(s - max(scores)) for s in scores]
    want = sum(wt * (Cv[t] @ BV) for t, wt in enumerate(w)) / sum(w)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # shifting every position by the same amount changes nothing
    shifted = O.attention_rope(q, Ck, Cv, BK, BV, 0.4, q_pos=T - 1 + 700, k_pos0=700)
    np.testing.assert_allclose(shifted, got, rtol=1e-9, atol=1e-12)
    # one token: the output is its value row whatever the rotation
    np.testing.assert_allclose(O.attention_rope(q, Ck[:1], Cv[:1], BK, BV, 0.4, q_pos=9), Cv[0] @ BV, atol=1e-12)


def test_latent_attention_rope_query_at_last_position():
    rng = np.random.default_rng(4)
    ranks, H = [8, 16], 16
    lens = [6, 0, 3]
    ck, cv = O.LatentCache(3, ranks, "i8", 32), O.LatentCache(3, ranks, "i8", 32)
    for b, L in enumerate(lens):
        ck.append(b, [O.quantize_i8(rng.standard_normal((L, r)).astype(np.float32)) for r in ranks])
        cv.append(b, [O.quantize_i8(rng.standard_normal((L, r)).astype(np.float32)) for r in ranks])
    BK = [rng.standard_normal((r, H)) for r in ranks]
    BV = [rng.standard_normal((r, H)) for r in ranks]
    q = rng.standard_normal((3, 2, H))
    out = O.latent_attention_rope(q, ck, cv, BK, BV, 0.25)
    assert np.all(out[1] == 0)
    for b in (0, 2):
        for h in range(2):
            want = O.attention_rope(q[b, h], ck.dequant(b, h), cv.dequant(b, h), BK[h], BV[h], 0.25, lens[b] - 1)
            np.testing.assert_array_equal(out[b, h], want)
            # at position 0 of a one-token-shorter window the scores differ: the query position matters
            other = O.attention_rope(q[b, h], ck.dequant(b, h), cv.dequant(b, h), BK[h], BV[h], 0.25, 0)
            assert not np.allclose(other, want)


# ---------------------------------------------------------------- hybrid linear split on output channels

def _outsplit_tiny():
    """K = 2 inputs, N = 3 outputs: output 1 dense, outputs 0 and 2 low-rank (R = 1)."""
    return dict(dense_out=[1], lr_out=[0, 2], W_D=np.array([[3], [1]], np.int8), s_D=np.array([0.25], np.float16),
                U=np.array([[3], [1]], np.int8), s_U=np.array([1.0], np.float16),
                V=np.array([[2, -1]], np.int8), s_V=np.array([0.5, 0.25], np.float16))


def test_outsplit_worked_example():
    """x = [2, -1], s_x = 0.5.  Dense output 1: (2*3 - 1*1) * 0.5 * 0.25 = 0.625.
    Latent: (2*3 - 1*1) * 0.5 * 1 = 2.5 -> s_t = fl32(2.5 / 127), code 127.
    Low-rank outputs: 127 * 2 * s_t * 0.5 and 127 * (-1) * s_t * 0.25."""
    x = np.array([[2, -1]], np.int8)
    y, t_q, s_t = O.linear_w8a8_outsplit(x, np.array([0.5], np.float32), **_outsplit_tiny())
    st = float(np.float32(2.5) / np.float32(127.0))
    assert t_q.tolist() == [[127]] and float(s_t[0]) == st
    np.testing.assert_array_equal(y[0], [127 * 2 * st * 0.5, 0.625, -127 * st * 0.25])
    # gate = this projection, up = a dense projection with hand-computed outputs [1, -0.5, 1]
    up = dict(dense_out=[0, 1, 2], lr_out=[], W_D=np.array([[1, 0, 1], [0, 1, 0]], np.int8),
              s_D=np.array([1.0, 1.0, 1.0], np.float16), U=None, s_U=None, V=None, s_V=None)
    m = O.ffn_gate_up_swiglu(x, np.array([0.5], np.float32), _outsplit_tiny(), up)
    g = y[0]
    want = [g[j] / (1.0 + math.exp(-g[j])) * u for j, u in enumerate([1.0, -0.5, 1.0])]
    np.testing.assert_allclose(m[0], want, rtol=1e-15)


def test_outsplit_reduces_to_the_input_split_at_the_extremes():
    """All outputs dense = the all-dense input split (a plain int8 GEMM); no
    outputs dense = the all-low-rank input split: the same numbers exactly."""
    rng = np.random.default_rng(21)
    M, K, N, R = 5, 64, 24, 16
    x = rng.integers(-127, 128, (M, K)).astype(np.int8)
    sx = (rng.random(M) * 0.01 + 0.001).astype(np.float32)
    W = rng.integers(-127, 128, (K, N)).astype(np.int8)
    sW = (rng.random(N) * 0.01 + 0.001).astype(np.float16)
    U = rng.integers(-127, 128, (K, R)).astype(np.int8)
    sU = (rng.random(R) * 0.01 + 0.001).astype(np.float16)
    V = rng.integers(-127, 128, (R, N)).astype(np.int8)
    sV = (rng.random(N) * 0.01 + 0.001).astype(np.float16)
    allc, none = list(range(N)), []
    y1, _, _ = O.linear_w8a8_outsplit(x, sx, allc, none, W, sW, U, sU, V, sV)
    y2, _, _ = O.linear_w8a8_hybrid(x, sx, list(range(K)), [], W, sW, None, None, None, None)
    np.testing.assert_array_equal(y1, y2)
    y3, tq3, st3 = O.linear_w8a8_outsplit(x, sx, none, allc, W, sW, U, sU, V, sV)
    y4, tq4, st4 = O.linear_w8a8_hybrid(x, sx, [], list(range(K)), None, None, U, sU, V, sV)
    np.testing.assert_array_equal(y3, y4)
    np.testing.assert_array_equal(tq3, tq4)
    # a split in between: each output channel equals the extreme it belongs to
    D = sorted(rng.choice(N, 6, replace=False).tolist())
    L = [j for j in range(N) if j not in D]
    y5, _, _ = O.linear_w8a8_outsplit(x, sx, D, L, W[:, D], sW[D], U, sU, V[:, L], sV[L])
    np.testing.assert_array_equal(y5[:, D], y1[:, D])
    np.testing.assert_array_equal(y5[:, L], y3[:, L])
