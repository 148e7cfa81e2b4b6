"""The two comparison points of the latent decode, against the oracle.

* lk_dense_decode_attn: flash-decoding over materialised bf16 K and V (the
  pages' baseline).  The oracle is attention_materialized with identity
  factors (B = I reproduces dense attention, a pinned special case), on the
  same bf16 values: 1e-5 * RMS for fp32 outputs, 1e-2 * RMS (plus half a
  bf16 ulp) for bf16 outputs.
* lk_latent_reconstruct_kv: the naive path's K = dequant(C_K) B_K and V,
  stored bf16: each value within one bf16 rounding of the oracle's float64
  product.  Attending them with the dense kernel matches the oracle's
  attention over its own bf16-rounded K and V within 1e-3 * RMS (a value
  whose fp32 sum straddles a bf16 rounding boundary may land one ulp off).
  Against the latent decode the naive path differs by what storing K and V
  in bf16 costs: float64 attention over bf16-rounded K, V moves these cases'
  outputs by up to 1.6% (int8 codes) and 2.7% (int4) of their RMS, so that
  comparison allows 4e-2 * RMS.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import assert_close_bf16, assert_close_rms, build_caches

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def _dense_case(B, nh, H, lens, cap, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, nh, H, generator=g).to(torch.bfloat16)
    K = (torch.randn(B, nh, cap, H, generator=g) * 0.7).to(torch.bfloat16)
    V = torch.randn(B, nh, cap, H, generator=g).to(torch.bfloat16)
    return q, K, V


def _oracle_dense(q, K, V, lens):
    B, nh, cap, H = K.shape
    out = np.zeros((B, nh, H))
    eye = np.eye(H)
    for b in range(B):
        for h in range(nh):
            if lens[b]:
                T = lens[b]
                out[b, h] = O.attention_materialized(q[b, h].double().numpy(), K[b, h, :T].double().numpy(),
                                                     V[b, h, :T].double().numpy(), eye, eye, 1.0 / math.sqrt(H))
    return out


@pytest.mark.parametrize("B,nh,H,lens,cap", [
    (2, 4, 128, [700, 33], 704),
    (1, 2, 128, [5000], 5008),           # many pieces per unit: the merge
    (3, 3, 64, [0, 1, 129], 144),        # empty row, single token, ragged
    (2, 2, 256, [300, 17], 304),         # two 16-byte chunks per lane
])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_dense_decode_matches_oracle(B, nh, H, lens, cap, out_dtype):
    lk = _lk()
    q, K, V = _dense_case(B, nh, H, lens, cap, seed=B * 100 + H)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = lk.dense_decode_attn(q.cuda(), K.cuda(), V.cuda(), seq, max(lens), out_dtype=out_dtype)
    torch.cuda.synchronize()
    lk.device_status()
    want = _oracle_dense(q, K, V, lens)
    got = out.float().cpu().numpy()
    if out_dtype == torch.float32:
        assert_close_rms(got, want, 1e-5, "dense fp32")
    else:
        assert_close_bf16(got, want, 1e-2, "dense bf16")
    for b in range(B):
        if lens[b] == 0:
            assert np.all(got[b] == 0)


@pytest.mark.parametrize("kind,ranks_k,ranks_v,group", [
    ("i8", [16, 32, 8, 64], [32, 8, 64, 16], 32),
    ("i8", [12, 20, 4, 36], [44, 60, 28, 52], 32),   # ranks not multiples of 16 (zero-padded k steps)
    ("i4", [24, 16, 32, 64], [16, 32, 24, 8], 32),   # one or two scale groups per token
    ("i4", [48, 16, 24, 64], [40, 8, 56, 16], 8),    # groups of 8: two groups inside each 16-dim step
    ("i4", [48, 24, 40, 64], [56, 8, 24, 16], 24),   # groups of 24 straddling the 16-dim steps
])
def test_reconstruct_then_dense_equals_latent(kind, ranks_k, ranks_v, group):
    lk = _lk()
    lens = [700, 33, 2049]
    B, H, cap = len(lens), 128, 2064
    rng = np.random.default_rng(5)
    lat_k = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_k] for b in range(B)]
    lat_v = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_v] for b in range(B)]
    ok, ov, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, kind, group)
    ck = lk.LatentCache(B, ranks_k, cap, kind, group)
    cv = lk.LatentCache(B, ranks_v, cap, kind, group, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(6)
    BK = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(torch.bfloat16)
    BV = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(torch.bfloat16)
    q = torch.randn(B, len(ranks_k), H, generator=g).to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    Kr, Vr = lk.reconstruct_kv(ck, cv, BK.cuda(), BV.cuda(), seq, max(lens), H)
    torch.cuda.synchronize()
    lk.device_status()
    offk = np.concatenate([[0], np.cumsum(ranks_k)])
    offv = np.concatenate([[0], np.cumsum(ranks_v)])
    BKf, BVf = BK.double().numpy(), BV.double().numpy()
    Kc, Vc = Kr.float().cpu().numpy(), Vr.float().cpu().numpy()
    nh = len(ranks_k)
    want_naive = np.zeros((B, nh, H))
    eye = np.eye(H)
    for b in range(B):
        for h in range(nh):
            T = lens[b]
            wk = ok.dequant(b, h) @ BKf[offk[h]:offk[h + 1]]
            wv = ov.dequant(b, h) @ BVf[offv[h]:offv[h + 1]]
            for got, want in ((Kc[b, h, :T], wk), (Vc[b, h, :T], wv)):
                # one bf16 rounding of an fp32 sum: |err| <= 2^-8 |value| + fp32 slack
                assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-5 * np.abs(want).max())
            kb = torch.from_numpy(wk).to(torch.bfloat16).double().numpy()
            vb = torch.from_numpy(wv).to(torch.bfloat16).double().numpy()
            want_naive[b, h] = O.attention_materialized(q[b, h].double().numpy(), kb, vb, eye, eye,
                                                        1.0 / math.sqrt(H))
    dense = lk.dense_decode_attn(q.cuda(), Kr, Vr, seq, max(lens), out_dtype=torch.float32)
    latent = lk.latent_decode_attn(ck, cv, q.cuda(), BK.cuda(), BV.cuda(), seq, max(lens), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_close_rms(dense.cpu().numpy(), want_naive, 1e-3, "naive path vs oracle on bf16 K, V")
    assert_close_rms(dense.cpu().numpy(), latent.cpu().numpy(), 4e-2, "naive path vs latent decode")
