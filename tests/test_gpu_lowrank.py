"""LASER hybrid W8A8 linear on the device vs the oracle.

The requantised low-rank latent t_q and its scale are bit-exact (exact int32
sums, fixed fp32 order); y is compared within 1e-5 * RMS (fp32 out) and
1e-2 * RMS (bf16 out).
"""
import numpy as np
import pytest
import torch

import oracle as O
from rank_latent_kv_lk_b200 import configs, synth
from tests.helpers import assert_close_bf16, assert_close_rms

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def make(k_in, n_out, rank, n_dense, m, seed, residual=False):
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(k_in, generator=g)
    D = torch.sort(perm[:n_dense]).values.to(torch.int32)
    notD = torch.sort(perm[n_dense:]).values.to(torch.int32)
    W_D, s_D = synth.int8_weight(g, n_out, n_dense)
    U, s_U = synth.int8_weight(g, rank, k_in - n_dense) if rank else (None, None)
    V, s_V = synth.int8_weight(g, n_out, rank) if rank else (None, None)
    x = torch.randn(m, k_in, generator=g) * 2
    xq, sx = O.quantize_rows_i8(x.numpy())
    res = torch.randn(m, n_out, generator=g).to(torch.bfloat16) if residual else None
    return dict(D=D, notD=notD, W_D=W_D, s_D=s_D, U=U, s_U=s_U, V=V, s_V=s_V, xq=xq, sx=sx, res=res,
                k_in=k_in, n_out=n_out, rank=rank)


def device_weight(c):
    lk = _lk()
    dev = lambda t: None if t is None else t.cuda()
    n_dense = c["D"].numel()
    return lk.LowrankWeight(c["k_in"], c["n_out"], c["rank"], dev(c["D"]) if n_dense else None,
                            dev(c["notD"]) if c["rank"] else None, dev(c["W_D"]) if n_dense else None,
                            dev(c["s_D"]) if n_dense else None, dev(c["U"]), dev(c["s_U"]), dev(c["V"]),
                            dev(c["s_V"]))


def oracle(c):
    T = lambda t: None if t is None else t.numpy().T
    return O.linear_w8a8_hybrid(c["xq"], c["sx"], c["D"].numpy(), c["notD"].numpy(), T(c["W_D"]),
                                c["s_D"].numpy(), T(c["U"]), None if c["s_U"] is None else c["s_U"].numpy(),
                                T(c["V"]), None if c["s_V"] is None else c["s_V"].numpy(),
                                residual=None if c["res"] is None else c["res"].float().numpy())


def run(c, y_dtype):
    lk = _lk()
    w = device_weight(c)
    m = c["xq"].shape[0]
    tq = torch.empty((m, c["rank"]), dtype=torch.int8, device="cuda") if c["rank"] else None
    ts = torch.empty((m,), dtype=torch.float32, device="cuda") if c["rank"] else None
    y = lk.lowrank_linear(w, torch.from_numpy(c["xq"]).cuda(), torch.from_numpy(c["sx"]).cuda(),
                          residual=None if c["res"] is None else c["res"].cuda(), y_dtype=y_dtype,
                          t_q_out=tq, t_scale_out=ts)
    torch.cuda.synchronize()
    lk.device_status()
    return y.float().cpu().numpy(), (None if tq is None else tq.cpu().numpy()), (None if ts is None else ts.cpu().numpy())


@pytest.mark.parametrize("y_dtype,tol", [(torch.float32, 1e-5), (torch.bfloat16, 1e-2)])
@pytest.mark.parametrize("shape", [(64, 40, 16, 16, 3), (256, 100, 32, 64, 1), (512, 77, 64, 128, 33)])
def test_small_shapes(shape, y_dtype, tol):
    c = make(*shape, seed=sum(shape), residual=True)
    y, tq, ts = run(c, y_dtype)
    yo, tqo, tso = oracle(c)
    assert np.array_equal(tq, tqo)
    assert np.array_equal(ts.view(np.uint32), tso.view(np.uint32))
    if y_dtype == torch.bfloat16:
        assert_close_bf16(y, yo, tol)
    else:
        assert_close_rms(y, yo, tol)


def test_all_dense_is_plain_w8a8_linear():
    c = make(256, 96, 0, 256, 5, seed=1)
    y, _, _ = run(c, torch.float32)
    assert_close_rms(y, oracle(c)[0], 1e-5)


def test_no_dense_is_pure_low_rank():
    c = make(128, 64, 32, 0, 4, seed=2)
    y, tq, _ = run(c, torch.float32)
    yo, tqo, _ = oracle(c)
    assert np.array_equal(tq, tqo)
    assert_close_rms(y, yo, 1e-5)


@pytest.mark.parametrize("which", ["gate", "down"])
def test_full_size_ffn_projection(which):
    """The hybrid FFN projections of the W8A8 layer workload at full size, 32 tokens."""
    w = configs.WORKLOADS[5]
    k_in, n_out = (w.embed_dim, w.ffn_inter) if which == "gate" else (w.ffn_inter, w.embed_dim)
    n_dense = int(round(w.ffn_dense_frac * k_in / 16)) * 16
    c = make(k_in, n_out, w.ffn_rank, n_dense, w.batch, seed=3 if which == "gate" else 4, residual=which == "down")
    y, tq, ts = run(c, torch.bfloat16)
    yo, tqo, tso = oracle(c)
    assert np.array_equal(tq, tqo)
    assert np.array_equal(ts.view(np.uint32), tso.view(np.uint32))
    assert_close_bf16(y, yo, 1e-2)
