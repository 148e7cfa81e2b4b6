"""One W8A8 decoder-layer decode step (latent attention + hybrid FFN) vs the oracle.

The context caches are filled with codes the oracle quantised from seeded
latents; the step then runs through the C ABI on the device and through
oracle.decoder_layer_w8a8 on the host from the same state.  Every
intermediate is compared: int8 activations by the band rule, bf16 tensors
within 1e-2 * RMS.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
from rank_latent_kv_lk_b200 import configs, synth
from rank_latent_kv_lk_b200.layer import W8A8DecoderLayer
from tests.helpers import assert_close_rms, build_caches

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def oracle_layer_dict(wts, n_heads, head_dim, rk, rv):
    T = lambda t: t.numpy().T

    def hyb(d):
        return dict(dense_idx=d["dense_idx"].numpy(), lr_idx=d["lr_idx"].numpy(), W_D=T(d["W_D"]),
                    s_D=d["s_D"].numpy(), U=T(d["U"]), s_U=d["s_U"].numpy(), V=T(d["V"]), s_V=d["s_V"].numpy())

    BK = wts["B_K"].float().numpy()
    BV = wts["B_V"].float().numpy()
    ok_ = np.concatenate([[0], np.cumsum(rk)])
    ov_ = np.concatenate([[0], np.cumsum(rv)])
    return dict(n_heads=n_heads, head_dim=head_dim, ranks_k=rk, ranks_v=rv,
                W_Q=T(wts["W_Q"]), s_Q=wts["s_Q"].numpy(), W_O=T(wts["W_O"]), s_O=wts["s_O"].numpy(),
                A=T(wts["A"]), s_A=wts["s_A"].numpy(),
                B_K=[BK[ok_[i]:ok_[i + 1]] for i in range(n_heads)],
                B_V=[BV[ov_[i]:ov_[i + 1]] for i in range(n_heads)],
                gate=hyb(wts["gate"]), up=hyb(wts["up"]), down=hyb(wts["down"]))


def run_layer(w, T_ctx, seed):
    rk, rv = [w.rank] * w.n_heads, [w.rank] * w.n_heads
    wts = synth.layer_weights_w8a8(w, rk, rv)
    capacity = (T_ctx + 1 + 15) // 16 * 16
    layer = W8A8DecoderLayer(wts, w.n_heads, w.head_dim, rk, rv, w.batch, capacity, w.ffn_inter)
    rng = np.random.default_rng(seed)
    lat_k = [[(rng.standard_normal((T_ctx, r)) * 1.5).astype(np.float32) for r in rk] for _ in range(w.batch)]
    lat_v = [[(rng.standard_normal((T_ctx, r)) * 1.5).astype(np.float32) for r in rv] for _ in range(w.batch)]
    ok, ov, (rows_k, sc_k), (rows_v, sc_v) = build_caches(lat_k, lat_v, rk, rv, "i8", 32)
    layer.cache_k.load(rows_k, sc_k)
    layer.cache_v.load(rows_v, sc_v)
    g = torch.Generator().manual_seed(seed + 1)
    x = torch.randn(w.batch, w.embed_dim, generator=g).to(torch.bfloat16)
    lens = [T_ctx] * w.batch
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    trace = {}
    out = layer.step(x.cuda(), seq, lens, trace)
    torch.cuda.synchronize()
    _lk().device_status()
    assert lens == [T_ctx + 1] * w.batch and seq.cpu().tolist() == lens
    want, inter = O.decoder_layer_w8a8(x.float().numpy(), oracle_layer_dict(wts, w.n_heads, w.head_dim, rk, rv),
                                       ok, ov)
    got = {k: (v.float().cpu().numpy() if torch.is_tensor(v) else v) for k, v in trace.items()}
    # int8 activations: the input of the first quantisation is exact, later ones are band-compared by value
    assert np.array_equal(got["xq"], inter["xq"])
    for name in ("q", "attn", "x2", "gate", "up"):
        assert_close_rms(got[name], inter[name], 1e-2, name)
    assert_close_rms(got["out"], want, 1e-2, "out")
    ffn_got = got["out"] - got["x2"]
    ffn_want = want - inter["x2"]
    assert_close_rms(ffn_got, ffn_want, 5e-2, "ffn delta")
    attn_delta = got["x2"] - x.float().numpy()
    assert_close_rms(attn_delta, inter["x2"] - x.float().numpy(), 5e-2, "attention delta")
    # the appended latents of the new token: the latent input x_q is exact, so bit-exact codes
    rows_k2, sc_k2 = layer.cache_k.read(lens)
    nk = sum(rk)
    for b in range(w.batch):
        for h, r in enumerate(rk):
            c, s = O.quantize_i8(inter["latent"][b:b + 1, sum(rk[:h]):sum(rk[:h]) + r])
            assert np.array_equal(rows_k2[b][h][-1:].view(np.int8), c)
            assert sc_k2[b][h][-1] == s[0]
    assert nk == sum(rk)


def test_layer_small():
    w = dataclasses.replace(configs.WORKLOADS[5], batch=4, embed_dim=256, n_heads=4, head_dim=64, rank=16,
                            ffn_inter=512, ffn_rank=64)
    run_layer(w, T_ctx=40, seed=31)


def test_layer_full_size():
    """B=32, E=4096, 32 heads x 128, r=32, context 4096, hybrid FFN 11008 (25% dense, rank 512)."""
    w = configs.WORKLOADS[5]
    run_layer(w, T_ctx=w.context, seed=32)
