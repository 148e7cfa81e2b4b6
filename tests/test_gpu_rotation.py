"""The outlier-smoothing rotations on the device against the oracle.

WSVD page, technical summary §2C: orthogonal S1 (a Hadamard matrix) on the
input and S2 on the latent smooth outlier channels before round-to-nearest.

* lk_rmsnorm_hadamard_quant_i8 (S1): codes and scales against the oracle's
  quantisation of its own fp32 RMSNorm(x) H_k, by the band rule (the device
  sums the butterflies in fp32; a code may differ by one only at a tie).
* a cache with rotation = 1 (S2 on append): codes against the oracle's
  quantisation of rotate_latents(x A), band rule, for every block order
  (ranks whose largest power-of-two divisor is 4 ... 64).
* decode over a rotated cache with the counter-rotated factors S2 B: the
  decode is the plain one, so the oracle is latent attention over the
  oracle-made rotated codes with S2 B, at the fp32 bound 1e-5 * RMS.
* the point of S2: on latents with a decaying per-dim magnitude (what
  A = U diag(sigma) gives) plus a few outlier dims, the device's rotated
  int8 and int4 caches reconstruct x A with a smaller error than the plain
  ones.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import assert_close_rms, build_caches, check_codes_band

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("m,k", [(37, 4096), (3, 64), (2, 1), (5, 16384)])
def test_rmsnorm_hadamard_quant_band(dtype, m, k):
    lk = _lk()
    g = torch.Generator().manual_seed(m + k)
    x = torch.randn(m, k, generator=g) * 2
    x[:, :: max(1, k // 8)] *= 25.0              # a few outlier channels
    x = x.to(dtype)
    q, s = lk.rmsnorm_hadamard_quant_i8(x.cuda(), 1e-5)
    torch.cuda.synchronize()
    y32 = O.rmsnorm_hadamard(x.float().numpy(), 1e-5).astype(np.float32)
    flips = check_codes_band(q.cpu().numpy(), s.cpu().numpy(), y32)
    assert flips <= max(3, m * k // 4000)


def test_hadamard_spreads_input_outliers():
    """S1's effect at the product entry point: int8 codes of RMSNorm(x) H,
    multiplied back by H, recover RMSNorm(x) better than the codes of
    RMSNorm(x) itself when x has outlier channels."""
    lk = _lk()
    g = torch.Generator().manual_seed(3)
    x = torch.randn(16, 4096, generator=g)
    x[:, torch.randperm(4096, generator=g)[:40]] *= 20.0
    y = O.rmsnorm(x.numpy(), 1e-5)
    q0, s0 = lk.rmsnorm_quant_i8(x.cuda(), 1e-5)
    q1, s1 = lk.rmsnorm_hadamard_quant_i8(x.cuda(), 1e-5)
    torch.cuda.synchronize()
    plain = q0.cpu().numpy().astype(np.float64) * s0.cpu().numpy()[:, None]
    rot = (q1.cpu().numpy().astype(np.float64) * s1.cpu().numpy()[:, None]) @ O.hadamard(4096)
    e_plain = np.sqrt(np.mean((plain - y) ** 2))
    e_rot = np.sqrt(np.mean((rot - y) ** 2))
    assert e_rot < 0.5 * e_plain, (e_rot, e_plain)


def _imbalanced_latents(rng, n, ranks, outlier=8.0):
    """Per head: dims with magnitude sigma_i = 1 / (1 + i / 4) (a decaying
    singular-value profile) and every 16th dim an outlier."""
    cols = []
    for r in ranks:
        sig = 1.0 / (1.0 + np.arange(r) / 4.0)
        sig[::16] *= outlier
        cols.append(rng.standard_normal((n, r)) * sig)
    return np.concatenate(cols, axis=1)


@pytest.mark.parametrize("kind", ["i8", "i4"])
def test_rotated_append_matches_oracle(kind):
    lk = _lk()
    # block orders 4 (r = 12, int8 only: int4 ranks are multiples of 8), 8, 16, 32, 64
    ranks_k = [12, 8, 24, 40, 16, 32, 48, 64] if kind == "i8" else [56, 8, 24, 40, 16, 32, 48, 64]
    ranks_v = list(reversed(ranks_k))
    B, E, cap = 2, 512, 128
    rng = np.random.default_rng(17)
    g = torch.Generator().manual_seed(17)
    A = (torch.randn(E, sum(ranks_k) + sum(ranks_v), generator=g) / math.sqrt(E))
    ck = lk.LatentCache(B, ranks_k, cap, kind, 32, rotation=True)
    cv = lk.LatentCache(B, ranks_v, cap, kind, 32, role="v", rotation=True)
    seq = torch.zeros(B, dtype=torch.int32, device="cuda")
    lens = [0] * B
    v_all = [[] for _ in range(B)]
    for n_new in (37, 1, 1):
        x = torch.from_numpy(rng.standard_normal((B * n_new, E))).float()
        lk.latent_project_append(ck, cv, x.cuda(), A.t().contiguous().cuda(), seq, lens)
        torch.cuda.synchronize()
        lk.device_status()
        v32 = O.latent_project_float(x.numpy(), A.numpy())
        vrot = O.rotate_latents(v32, ranks_k + ranks_v)
        for b in range(B):
            v_all[b].append(vrot[b * n_new:(b + 1) * n_new])
        lens = [L + n_new for L in lens]
    assert seq.cpu().tolist() == lens
    flips = 0
    for b in range(B):
        v = np.concatenate(v_all[b])
        off = 0
        for cache, ranks in ((ck, ranks_k), (cv, ranks_v)):
            for h, r in enumerate(ranks):
                rows, sc = cache.read_unit(b, h, lens[b])
                codes = rows.view(np.int8) if kind == "i8" else O.unpack_i4(rows, r)
                flips += check_codes_band(codes, sc, v[:, off:off + r], kind, min(32, r))
                off += r
    assert flips <= 40


@pytest.mark.parametrize("kind", ["i8", "i4"])
def test_rotated_cache_decode_with_counter_rotated_factors(kind):
    lk = _lk()
    ranks_k, ranks_v = [16, 48, 8, 64], [64, 24, 32, 16]
    lens = [700, 33, 1500]
    B, H, cap = len(lens), 128, 1504
    rng = np.random.default_rng(23)
    lat_k = [[O.rotate_latents(_imbalanced_latents(rng, lens[b], [r]), [r]) for r in ranks_k] for b in range(B)]
    lat_v = [[O.rotate_latents(_imbalanced_latents(rng, lens[b], [r]), [r]) for r in ranks_v] for b in range(B)]
    ok, ov, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, kind, 32)
    ck = lk.LatentCache(B, ranks_k, cap, kind, 32, rotation=True)
    cv = lk.LatentCache(B, ranks_v, cap, kind, 32, role="v", rotation=True)
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(24)
    BK_h = [torch.randn(r, H, generator=g).double().numpy() / math.sqrt(r) for r in ranks_k]
    BV_h = [torch.randn(r, H, generator=g).double().numpy() / math.sqrt(r) for r in ranks_v]
    # counter-rotated factors S2 B, stored fp32 (the oracle uses the same fp32 values)
    SBK = [(O.latent_rotation(r) @ b).astype(np.float32) for r, b in zip(ranks_k, BK_h)]
    SBV = [(O.latent_rotation(r) @ b).astype(np.float32) for r, b in zip(ranks_v, BV_h)]
    q = torch.randn(B, len(ranks_k), H, generator=g)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = lk.latent_decode_attn(ck, cv, q.cuda(), torch.from_numpy(np.concatenate(SBK)).cuda(),
                                torch.from_numpy(np.concatenate(SBV)).cuda(), seq, max(lens),
                                out_dtype=torch.float32)
    torch.cuda.synchronize()
    lk.device_status()
    want = O.latent_attention(q.double().numpy(), ok, ov, SBK, SBV, 1.0 / math.sqrt(H))
    assert_close_rms(out.cpu().numpy(), want, 1e-5, "decode over a rotated cache")


@pytest.mark.parametrize("kind", ["i8", "i4"])
def test_rotation_lowers_latent_quantisation_error(kind):
    lk = _lk()
    ranks = [64, 48, 32, 16]
    B, n, cap = 1, 256, 256
    rng = np.random.default_rng(31)
    v = _imbalanced_latents(rng, B * n, ranks).astype(np.float32)
    E = sum(ranks)
    # x = v, A = I: the appended latent is exactly v
    x = torch.from_numpy(v)
    A = torch.eye(E)
    errs = {}
    for rot in (False, True):
        ck = lk.LatentCache(B, ranks, cap, kind, 32, rotation=rot)
        cv = lk.LatentCache(B, ranks, cap, kind, 32, role="v", rotation=rot)
        seq = torch.zeros(B, dtype=torch.int32, device="cuda")
        lk.latent_project_append(ck, cv, x.cuda(), torch.cat([A, A]).contiguous().cuda(), seq, [0])
        torch.cuda.synchronize()
        lk.device_status()
        sq, off = 0.0, 0
        for h, r in enumerate(ranks):
            rows, sc = ck.read_unit(0, h, n)
            if kind == "i8":
                deq = rows.view(np.int8).astype(np.float64) * sc.astype(np.float64)[:, None]
            else:
                codes = O.unpack_i4(rows, r)
                idx = np.arange(r) // min(32, r)
                deq = codes.astype(np.float64) * sc.astype(np.float64)[:, idx]
            if rot:
                deq = deq @ O.latent_rotation(r).T
            sq += float(np.sum((deq - v[:, off:off + r]) ** 2))
            off += r
        errs[rot] = math.sqrt(sq / v.size)
    print(f"{kind}: latent RTN error {errs[False]:.3e} plain, {errs[True]:.3e} rotated")
    assert errs[True] < 0.8 * errs[False], errs
