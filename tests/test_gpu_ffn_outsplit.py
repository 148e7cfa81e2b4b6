"""The FFN input side split on output channels (gate + up + SwiGLU), device
against oracle.ffn_gate_up_swiglu.

The int32 sums are exact on both sides and the low-rank latent is
requantised from identically rounded fp32 values, so the latent codes agree
exactly; the outputs differ only by the device's fp32 scaling and SwiGLU
(two fp32 roundings of each projection, expf): within 1e-5 * RMS of the
oracle's float64 values.  Small cases run whole (several token-row chunks,
ragged channel tiles, all-dense and all-low-rank splits); the workload-5
size (B = 32, E = 4096, hidden 11008, 25 % dense, rank 512) is checked on a
seeded sample of 384 hidden channels, the oracle run on just those."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
from rank_latent_kv_lk_b200 import synth
from rank_latent_kv_lk_b200.configs import WORKLOADS
from tests.helpers import assert_close_rms

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def _x(m, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.clamp(torch.round(torch.randn(m, k, generator=g) * 40), -127, 127).to(torch.int8)
    s = (torch.rand(m, generator=g) * 0.01 + 0.002).to(torch.float32)
    return x, s


def _oracle_args(d, name, cols=None):
    """Oracle weight arguments (input-major) for projection `name`, optionally
    restricted to the hidden channels `cols` (renumbered 0..len(cols)-1)."""
    w = {k: v.numpy() for k, v in d[name].items()}
    dense = d["dense_out"].numpy()
    lr = d["lr_out"].numpy()
    if cols is None:
        cols = np.arange(d["n_out"])
    pos = {int(c): i for i, c in enumerate(cols)}
    di = [i for i, c in enumerate(dense) if int(c) in pos]
    li = [i for i, c in enumerate(lr) if int(c) in pos]
    return dict(dense_out=[pos[int(dense[i])] for i in di], lr_out=[pos[int(lr[i])] for i in li],
                W_D=w["W_D"][di].T, s_D=w["s_D"][di], U=w["U"].T, s_U=w["s_U"],
                V=w["V"][li].T, s_V=w["s_V"][li])


@pytest.mark.parametrize("m,k_in,n_out,rank,frac", [
    (1, 256, 200, 64, 0.25),
    (5, 512, 184, 32, 0.5),
    (32, 256, 136, 64, 0.25),
    (40, 128, 96, 16, 0.25),      # two token-row chunks
    (7, 256, 160, 0, 1.0),        # every channel dense
    (3, 256, 120, 48, 0.0),       # every channel low-rank
])
def test_ffn_outsplit_matches_oracle(m, k_in, n_out, rank, frac):
    lk = _lk()
    w = WORKLOADS[5]
    d = synth.ffn_outsplit_weights(w, k_in=k_in, n_out=n_out, rank=max(rank, 16), dense_frac=frac)
    if frac == 1.0:
        d["rank"] = 0
    x, s = _x(m, k_in, seed=m * 31 + n_out)
    ffn = lk.OutsplitFfn(d)
    out = ffn(x.cuda(), s.cuda())
    torch.cuda.synchronize()
    lk.device_status()
    want = O.ffn_gate_up_swiglu(x.numpy(), s.numpy(), _oracle_args(d, "gate"), _oracle_args(d, "up"))
    assert_close_rms(out.cpu().numpy(), want, 1e-5, "ffn gate+up+swiglu")


def test_ffn_outsplit_workload5_size_sampled():
    lk = _lk()
    w = WORKLOADS[5]
    d = synth.ffn_outsplit_weights(w)
    x, s = _x(w.batch, w.embed_dim, seed=55)
    ffn = lk.OutsplitFfn(d)
    out = ffn(x.cuda(), s.cuda())
    torch.cuda.synchronize()
    lk.device_status()
    cols = np.sort(np.random.default_rng(56).choice(d["n_out"], 384, replace=False))
    want = O.ffn_gate_up_swiglu(x.numpy(), s.numpy(), _oracle_args(d, "gate", cols), _oracle_args(d, "up", cols))
    assert_close_rms(out.cpu().numpy()[:, cols], want, 1e-5, "ffn gate+up+swiglu, workload 5 size")
