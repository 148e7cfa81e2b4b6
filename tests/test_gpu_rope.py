"""Rotary-position latent decode on the device against the oracle.

* lk_rope_table: every (cos, sin) entry equals the float64 value rounded to
  fp32, within one fp32 ulp (the device evaluates the same float64 formula).
* lk_latent_decode_attn_rope: caches built by the oracle (codes and scales
  from its quantiser), loaded into the device layout; the output against
  oracle.latent_attention_rope (keys rebuilt and rotated in float64, query at
  the newest position of each row) within 1e-5 * RMS for fp32 outputs (the
  device rebuilds keys from exact bf16 products summed in fp32 and rotates
  with fp32 table values) and 1e-2 * RMS plus half a bf16 ulp for bf16
  outputs.  Cases: int8 and int4 (one and several scale groups, groups that
  straddle the 16-dim product steps), ranks not multiples of 16, ragged
  lengths with empty and one-token rows, several 128-token tiles and pieces
  per (b, h), head dims 64, 128 and 256.
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


@pytest.mark.parametrize("H,max_pos", [(128, 20000), (64, 300), (256, 1000)])
def test_rope_table_matches_float64(H, max_pos):
    lk = _lk()
    tab = lk.rope_table(H, max_pos).cpu().numpy()
    ang = O.rope_angles(np.arange(max_pos), H)
    for k, f in ((0, np.cos), (1, np.sin)):
        want = f(ang).astype(np.float32)
        got = tab[:, :, k]
        ulp = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
        # values of opposite sign near zero: compare by magnitude instead
        close = np.abs(got - want) <= 2.0 ** -24
        assert np.all((ulp <= 1) | close), f"{'cos' if k == 0 else 'sin'} off by {ulp.max()} ulp"


CASES = [
    # kind, ranks_k, ranks_v, group, lens, H, q dtype
    ("i8", [32, 64, 16, 8], [16, 32, 64, 24], 32, [3000, 1, 0, 517], 128, torch.bfloat16),
    ("i8", [12, 20, 36, 4], [44, 60, 28, 52], 32, [700, 129], 128, torch.float32),
    ("i8", [64], [64], 32, [16385], 128, torch.bfloat16),                 # one long row: many pieces
    ("i4", [24, 16, 32, 64], [16, 32, 24, 8], 32, [1500, 33, 260], 128, torch.bfloat16),
    ("i4", [48, 16, 24, 64], [40, 8, 56, 16], 8, [900, 2], 64, torch.bfloat16),
    ("i4", [48, 24, 40, 64], [56, 8, 24, 16], 24, [640, 127], 256, torch.float32),
]


@pytest.mark.parametrize("kind,ranks_k,ranks_v,group,lens,H,qdt", CASES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_rope_decode_matches_oracle(kind, ranks_k, ranks_v, group, lens, H, qdt, out_dtype):
    lk = _lk()
    B, nh = len(lens), len(ranks_k)
    cap = (max(lens) + 16 + 15) // 16 * 16
    rng = np.random.default_rng(sum(lens) + H)
    lat_k = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_k] for b in range(B)]
    lat_v = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks_v] for b in range(B)]
    ok, ov, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, kind, group)
    ck = lk.LatentCache(B, ranks_k, cap, kind, group)
    cv = lk.LatentCache(B, ranks_v, cap, kind, group, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(B * 7 + H)
    BK = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(torch.bfloat16)
    BV = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(torch.bfloat16)
    q = torch.randn(B, nh, H, generator=g).to(qdt)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    table = lk.rope_table(H, cap)
    out = lk.latent_decode_attn_rope(ck, cv, q.cuda(), BK.cuda(), BV.cuda(), seq, max(lens), table,
                                     out_dtype=out_dtype)
    out2 = lk.latent_decode_attn_rope(ck, cv, q.cuda(), BK.cuda(), BV.cuda(), seq, max(lens), table,
                                      out_dtype=out_dtype)  # the counters were left zero
    torch.cuda.synchronize()
    lk.device_status()
    offk = np.concatenate([[0], np.cumsum(ranks_k)])
    offv = np.concatenate([[0], np.cumsum(ranks_v)])
    BKh = [BK.double().numpy()[offk[h]:offk[h + 1]] for h in range(nh)]
    BVh = [BV.double().numpy()[offv[h]:offv[h + 1]] for h in range(nh)]
    want = O.latent_attention_rope(q.double().numpy(), ok, ov, BKh, BVh, 1.0 / math.sqrt(H))
    got = out.float().cpu().numpy()
    assert np.array_equal(got, out2.float().cpu().numpy()), "the result depends on the call"
    if out_dtype == torch.float32:
        assert_close_rms(got, want, 1e-5, "rope decode fp32")
    else:
        assert_close_bf16(got, want, 1e-2, "rope decode bf16")
    for b in range(B):
        if lens[b] == 0:
            assert np.all(got[b] == 0)


def test_rope_decode_differs_from_plain_decode():
    """The rotation matters: on the same caches the rotary output is not the
    plain (absorbed) one, while a one-token row gives that token's value row
    either way."""
    lk = _lk()
    ranks = [32, 32]
    lens = [400, 1]
    B, H, cap = 2, 128, 416
    rng = np.random.default_rng(11)
    lat = [[(rng.standard_normal((lens[b], r)) * 1.3).astype(np.float32) for r in ranks] for b in range(B)]
    ok, ov, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat, lat, ranks, ranks, "i8", 32)
    ck = lk.LatentCache(B, ranks, cap, "i8", 32)
    cv = lk.LatentCache(B, ranks, cap, "i8", 32, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(12)
    BK = (torch.randn(64, H, generator=g) / 6).to(torch.bfloat16).cuda()
    BV = (torch.randn(64, H, generator=g) / 6).to(torch.bfloat16).cuda()
    q = torch.randn(B, 2, H, generator=g).to(torch.bfloat16).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    rot = lk.latent_decode_attn_rope(ck, cv, q, BK, BV, seq, max(lens), lk.rope_table(H, cap),
                                     out_dtype=torch.float32)
    plain = lk.latent_decode_attn(ck, cv, q, BK, BV, seq, max(lens), out_dtype=torch.float32)
    torch.cuda.synchronize()
    r, p = rot.cpu().numpy(), plain.cpu().numpy()
    assert np.abs(r[0] - p[0]).max() > 1e-2 * np.abs(p[0]).max()
    np.testing.assert_allclose(r[1], p[1], rtol=1e-5, atol=1e-6)
