"""Latent decode attention on the device vs the oracle (K and V materialised).

Caches are filled with codes the oracle quantised from seeded latents, so the
device and the oracle read the same cache; only the attention arithmetic is
compared.  Tolerances: 1e-5 * RMS for fp32 outputs, 1e-2 * RMS for bf16.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from rank_latent_kv_lk_b200 import configs, synth
from tests.helpers import assert_close_bf16, assert_close_rms, build_caches

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def make_case(B, ranks_k, ranks_v, H, lens, kind="i8", group=32, capacity=None, seed=0,
              dtype=torch.bfloat16, live_rows=None, sigma=1.3):
    """Device caches + factors + q, and the oracle's caches over the same codes.

    Rows outside live_rows hold all-zero latents (zero codes and scales)."""
    lk = _lk()
    rng = np.random.default_rng(seed)
    capacity = capacity or max(16, (max(lens) + 15) // 16 * 16)
    live = set(range(B)) if live_rows is None else set(live_rows)
    lat_k, lat_v = [], []
    for b in range(B):
        T = lens[b]
        mk = (lambda r: (rng.standard_normal((T, r)) * sigma).astype(np.float32)) if b in live else \
            (lambda r: np.zeros((T, r), np.float32))
        lat_k.append([mk(r) for r in ranks_k])
        lat_v.append([mk(r) for r in ranks_v])
    ok, ov, (rk_rows, rk_sc), (rv_rows, rv_sc) = build_caches(lat_k, lat_v, ranks_k, ranks_v, kind, group)
    ck = lk.LatentCache(B, ranks_k, capacity, kind, group)
    cv = lk.LatentCache(B, ranks_v, capacity, kind, group, role="v")
    ck.load(rk_rows, rk_sc)
    cv.load(rv_rows, rv_sc)
    g = torch.Generator().manual_seed(seed + 1)
    q = torch.randn(B, len(ranks_k), H, generator=g).to(dtype)
    BK = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_k]).to(dtype)
    BV = torch.cat([torch.randn(r, H, generator=g) / math.sqrt(r) for r in ranks_v]).to(dtype)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return dict(ck=ck, cv=cv, ok=ok, ov=ov, q=q, BK=BK, BV=BV, seq=seq, lens=lens, ranks_k=ranks_k,
                ranks_v=ranks_v, H=H)


def oracle_out(c, rows=None):
    q = c["q"].float().numpy()
    BK, BV = c["BK"].float().numpy(), c["BV"].float().numpy()
    offk = np.concatenate([[0], np.cumsum(c["ranks_k"])])
    offv = np.concatenate([[0], np.cumsum(c["ranks_v"])])
    BKh = [BK[offk[i]:offk[i + 1]] for i in range(len(c["ranks_k"]))]
    BVh = [BV[offv[i]:offv[i + 1]] for i in range(len(c["ranks_v"]))]
    scale = 1.0 / math.sqrt(c["H"])
    B, nh, H = q.shape
    out = np.zeros((B, nh, H))
    for b in (range(B) if rows is None else rows):
        for h in range(nh):
            if c["lens"][b] == 0:
                continue
            out[b, h] = O.attention_materialized(q[b, h], c["ok"].dequant(b, h), c["ov"].dequant(b, h),
                                                 BKh[h], BVh[h], scale)
    return out


def check(got, want, out_dtype, what):
    if out_dtype == torch.bfloat16:
        return assert_close_bf16(got, want, 1e-2, what)
    return assert_close_rms(got, want, 1e-5, what)


def run(c, out_dtype=torch.float32, n_split=0):
    lk = _lk()
    out = lk.latent_decode_attn(c["ck"], c["cv"], c["q"].cuda(), c["BK"].cuda(), c["BV"].cuda(), c["seq"],
                                max(c["lens"]), out_dtype=out_dtype, n_split=n_split)
    torch.cuda.synchronize()
    lk.device_status()
    return out.float().cpu().numpy()


def test_fp32_single_layer_shape():
    w = configs.WORKLOADS[1]
    c = make_case(1, [16] * 8, [16] * 8, 64, [257], capacity=w.capacity, dtype=torch.float32, seed=1)
    assert_close_rms(run(c), oracle_out(c), 1e-5, "fp32")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_ragged_ranks_and_lengths(out_dtype):
    c = make_case(5, [8, 16, 32, 48, 64, 8], [64, 8, 16, 48, 32, 16], 128, [0, 1, 17, 130, 300], seed=2)
    got = run(c, out_dtype)
    want = oracle_out(c)
    assert np.all(got[0] == 0)  # empty row
    check(got, want, out_dtype, "ragged")


@pytest.mark.parametrize("r,g,lens", [(24, 32, [1000, 16, 1]), (64, 16, [300, 129, 2]), (16, 8, [77, 5, 64])])
def test_int4_groups(r, g, lens):
    c = make_case(3, [r] * 4, [r] * 4, 128, lens, kind="i4", group=g, seed=3 + r)
    assert_close_rms(run(c), oracle_out(c), 1e-5, "int4")


def test_head_dim_64_and_odd_heads():
    c = make_case(2, [32, 16, 8], [8, 32, 64], 64, [200, 513], seed=4)
    assert_close_rms(run(c), oracle_out(c), 1e-5, "H=64")


@pytest.mark.parametrize("n_split", [1, 2, 7, 0, 1000])
def test_split_count_does_not_change_result(n_split):
    c = make_case(2, [32] * 4, [32] * 4, 128, [2000, 1234], seed=5)
    want = oracle_out(c)
    got = run(c, n_split=n_split)
    assert_close_rms(got, want, 1e-5, f"split {n_split}")


def test_workspace_counters_left_zero():
    lk = _lk()
    c = make_case(2, [32] * 4, [32] * 4, 128, [1500, 700], seed=6)
    run(c, n_split=5)
    ws = lk.workspaces.get("decode", 0, "cuda:0")
    assert int(ws[: 2 * 4 * 4].view(torch.int32).abs().sum().item()) == 0
    # a second call on the same workspace gives the same result
    assert_close_rms(run(c, n_split=5), oracle_out(c), 1e-5, "second call")


def test_uniform_scores_give_mean_of_v():
    """Closed form on the device: q = 0 gives the mean of V."""
    c = make_case(1, [16] * 2, [16] * 2, 64, [333], seed=7, dtype=torch.float32)
    c["q"] = torch.zeros_like(c["q"])
    got = run(c)
    BV = c["BV"].float().numpy()
    for h in range(2):
        mean_lat = c["ov"].dequant(0, h).mean(axis=0)
        np.testing.assert_allclose(got[0, h], mean_lat @ BV[16 * h:16 * (h + 1)], rtol=0, atol=1e-5)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_llava_shape_full(out_dtype):
    """B=1, 32 heads x H=128, r=32 int8, T=4097 (the first decode step of the 4096-token context)."""
    w = configs.WORKLOADS[2]
    c = make_case(1, [32] * 32, [32] * 32, 128, [w.context + 1], capacity=w.capacity, seed=8)
    check(run(c, out_dtype), oracle_out(c), out_dtype, "llava")


def test_int4_batch16_full_launch_sampled_rows():
    """B=16, 32 heads, r=24 int4 (group 32 -> 24), T=8193: all rows launched, rows 3 and 12 compared
    against the oracle, the all-zero rows must give zero output."""
    w = configs.WORKLOADS[3]
    lens = [w.context + 1] * w.batch
    c = make_case(w.batch, [24] * 32, [24] * 32, 128, lens, kind="i4", group=32, capacity=w.capacity,
                  seed=9, live_rows=[3, 12])
    got = run(c, torch.bfloat16)
    want = oracle_out(c, rows=[3, 12])
    for b in (3, 12):
        assert_close_bf16(got[b], want[b], 1e-2, f"row {b}")
    others = [b for b in range(w.batch) if b not in (3, 12)]
    assert np.all(got[others] == 0)


def test_ragged_layer_full_launch_sampled_rows():
    """One layer of the ragged-rank workload at full size: B=8, 32 heads with drawn ranks, T=16385."""
    w = configs.WORKLOADS[4]
    rk, rv = synth.ranks(w)
    lens = [w.context + 1] * w.batch
    c = make_case(w.batch, rk[0], rv[0], 128, lens, capacity=w.capacity, seed=10, live_rows=[0, 5])
    got = run(c, torch.bfloat16)
    want = oracle_out(c, rows=[0, 5])
    for b in (0, 5):
        assert_close_bf16(got[b], want[b], 1e-2, f"row {b}")
