"""Latent projection + quantise + append on the device vs the oracle.

Float inputs: the device sums x A^T in fp32 in its own order, so a code may
differ by one only at a rounding tie (band rule, tests/helpers.py).  int8
inputs: the int32 sum is exact and the dequantisation order is fixed, so codes
and scales are bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
from rank_latent_kv_lk_b200 import configs, synth
from tests.helpers import check_codes_band

pytestmark = pytest.mark.gpu


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


class Harness:
    def __init__(self, B, ranks_k, ranks_v, capacity, kind="i8", group=32):
        lk = _lk()
        self.B, self.rk, self.rv, self.kind, self.group = B, ranks_k, ranks_v, kind, group
        self.ck = lk.LatentCache(B, ranks_k, capacity, kind, group)
        self.cv = lk.LatentCache(B, ranks_v, capacity, kind, group, role="v")
        self.seq = torch.zeros(B, dtype=torch.int32, device="cuda")
        self.lens = [0] * B
        self.v_oracle = [[] for _ in range(B)]  # per row: list of float32 [n, N_tot]

    def append(self, x, A, v32, x_scale=None, a_scale=None):
        """x: [B * n_new, E] device; v32: oracle latents [B * n_new, N_tot]."""
        lk = _lk()
        n_new = x.shape[0] // self.B
        lk.latent_project_append(self.ck, self.cv, x, A, self.seq, self.lens, x_scale, a_scale)
        torch.cuda.synchronize()
        lk.device_status()
        for b in range(self.B):
            self.v_oracle[b].append(v32[b * n_new:(b + 1) * n_new])
        self.lens = [L + n_new for L in self.lens]
        assert self.seq.cpu().tolist() == self.lens

    def check(self, exact=False):
        nk = sum(self.rk)
        rows_k, sc_k = self.ck.read(self.lens)
        rows_v, sc_v = self.cv.read(self.lens)
        flips = 0
        for b in range(self.B):
            v = np.concatenate(self.v_oracle[b])
            off = 0
            for which, ranks, rows, sc in (("k", self.rk, rows_k, sc_k), ("v", self.rv, rows_v, sc_v)):
                for h, r in enumerate(ranks):
                    vh = v[:, off:off + r]
                    off += r
                    if self.kind == "i8":
                        codes = rows[b][h].view(np.int8)
                        g = r
                    else:
                        codes = O.unpack_i4(rows[b][h], r)
                        g = min(self.group, r)
                    if exact:
                        if self.kind == "i8":
                            oc, os_ = O.quantize_i8(vh)
                            assert np.array_equal(codes, oc), (which, b, h)
                            assert np.array_equal(sc[b][h].view(np.uint32), os_.view(np.uint32))
                        else:
                            oc, os_ = O.quantize_i4(vh, g)
                            assert np.array_equal(codes, oc), (which, b, h)
                            assert np.array_equal(sc[b][h].view(np.uint16), os_.view(np.uint16))
                    else:
                        flips += check_codes_band(codes, sc[b][h], vh, self.kind, g)
            assert off == v.shape[1]
        return flips


def _float_case(w, B, n_prefill, n_decode, ranks_k, ranks_v, seed):
    g = torch.Generator().manual_seed(seed)
    dt = synth.act_dtype(w)
    E = w.embed_dim
    A, _, _ = synth.factors(w, 0, ranks_k, ranks_v)
    h = Harness(B, ranks_k, ranks_v, w.capacity, w.kind, w.group)
    A_dev = A.cuda()
    A64 = A.float().numpy().T
    calls = [n_prefill] + [1] * n_decode
    for n in calls:
        x = torch.randn(B * n, E, generator=g).to(dt)
        v32 = O.latent_project_float(x.float().numpy(), A64)
        h.append(x.cuda(), A_dev, v32)
    return h


def test_fp32_prefill_and_decode():
    w = configs.WORKLOADS[1]
    h = _float_case(w, 1, 256, 1, [16] * 8, [16] * 8, seed=11)
    assert h.lens == [257]
    assert h.check() <= 20


def test_bf16_prefill_then_decode_steps():
    w = configs.WORKLOADS[2]
    h = _float_case(w, 2, 100, 2, [32] * 32, [32] * 32, seed=12)
    assert h.check() <= 40


def test_int4_cache_append():
    w = configs.WORKLOADS[3]
    h = _float_case(w, 3, 50, 1, [24] * 32, [24] * 32, seed=13)
    assert h.check() <= 40


def test_ragged_ranks_append():
    w = configs.WORKLOADS[4]
    rk, rv = synth.ranks(w)
    h = _float_case(w, 2, 40, 1, rk[0], rv[0], seed=14)
    assert h.check() <= 40


@pytest.mark.parametrize("B", [1, 8, 9, 16, 32, 64, 65])
def test_decode_rows_gemv(B):
    w = configs.WORKLOADS[2]
    h = _float_case(w, B, 1, 1, [32] * 32, [32] * 32, seed=15 + B)
    # codes off by one only inside the rounding band (check() raises
    # otherwise); their count grows with the rows: about 20 per 32 rows
    assert h.check() <= 20 * max(1, -(-B // 32))


def _w8a8_case(B, n_prefill, n_decode, seed):
    w = configs.WORKLOADS[5]
    rk, rv = [32] * 32, [32] * 32
    wts = synth.layer_weights_w8a8(w, rk, rv)
    A_q, s_A = wts["A"], wts["s_A"]
    h = Harness(B, rk, rv, 256)
    g = torch.Generator().manual_seed(seed)
    A_dev, sA_dev = A_q.cuda(), s_A.cuda()
    for n in [n_prefill] + [1] * n_decode:
        x = torch.randn(B * n, w.embed_dim, generator=g) * 2
        xq, sx = O.quantize_rows_i8(x.numpy())
        v32 = O.latent_project_w8a8(xq, sx, A_q.numpy().T, s_A.numpy())
        h.append(torch.from_numpy(xq).cuda(), A_dev, v32, torch.from_numpy(sx).cuda(), sA_dev)
    return h


def test_w8a8_append_bit_exact():
    h = _w8a8_case(4, 64, 2, seed=21)
    h.check(exact=True)


def test_capacity_overflow_writes_nothing():
    lk = _lk()
    w = configs.WORKLOADS[1]
    h = _float_case(w, 1, 256, 0, [16] * 8, [16] * 8, seed=22)
    before = (h.ck.codes.clone(), h.ck.scales.clone(), h.seq.clone())
    A, _, _ = synth.factors(w, 0, [16] * 8, [16] * 8)
    x = torch.randn(17, w.embed_dim, dtype=torch.float32, device="cuda")
    with pytest.raises(lk.LkError) as ei:
        lk.latent_project_append(h.ck, h.cv, x, A.cuda(), h.seq, h.lens)
    assert ei.value.status == 5  # LK_ERR_CAPACITY
    torch.cuda.synchronize()
    assert torch.equal(before[0], h.ck.codes) and torch.equal(before[1], h.ck.scales)
    assert torch.equal(before[2], h.seq)
