"""Device quantisers vs the oracle: bit-exact on identical float32 inputs."""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from tests.helpers import check_codes_band, to_dev

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _lk():
    import rank_latent_kv_lk_b200 as lk
    return lk


def _adversarial_rows(r, rng):
    """Rows that hit ties, zero, subnormals, saturation and a single non-zero."""
    rows = []
    e = -3
    s = 2.0 ** e
    row = np.zeros(r, np.float32)
    row[0] = 127 * s
    row[1:] = ((np.arange(1, r) % 9) - 4 + 0.5) * s  # exact half-integer ratios
    rows.append(row)
    rows.append(np.zeros(r, np.float32))
    sub = np.zeros(r, np.float32)
    sub[:4] = np.array([190, 95, -190, 3], np.float64) * 2.0 ** -149
    rows.append(sub.astype(np.float32))
    one = np.zeros(r, np.float32)
    one[r // 2] = -3.0
    rows.append(one)
    eqm = np.zeros(r, np.float32)
    eqm[0], eqm[1] = 5.0, -5.0
    rows.append(eqm)
    rows.append((rng.standard_normal(r) * 1e-30).astype(np.float32))
    rows.append((rng.standard_normal(r) * 1e30).astype(np.float32))
    return np.stack(rows)


@pytest.mark.parametrize("r", [4, 8, 16, 24, 32, 48, 64])
def test_quantize_latent_i8_bit_exact(r):
    lk = _lk()
    rng = np.random.default_rng(r)
    v = np.concatenate([(rng.standard_normal((997, r)) * rng.uniform(1e-3, 1e3, (997, 1))).astype(np.float32),
                        _adversarial_rows(r, rng)])
    c, s = lk.quantize_latent(to_dev(v), "i8")
    oc, os_ = O.quantize_i8(v)
    assert np.array_equal(c.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("r,g", [(8, 8), (16, 8), (24, 32), (24, 8), (48, 32), (64, 16), (64, 64), (12, 8)])
def test_quantize_latent_i4_bit_exact(r, g):
    lk = _lk()
    rng = np.random.default_rng(100 + r + g)
    v = np.concatenate([(rng.standard_normal((1001, r)) * rng.uniform(1e-3, 1e3, (1001, 1))).astype(np.float32),
                        _adversarial_rows(r, rng),
                        np.full((1, r), 7e6, np.float32)])
    c, s = lk.quantize_latent(to_dev(v), "i4", g)
    oc, os_ = O.quantize_i4(v, min(g, r))
    assert np.array_equal(c.cpu().numpy(), O.pack_i4(oc))
    assert np.array_equal(s.cpu().numpy().view(np.uint16), os_.view(np.uint16))


def test_quantize_golden_fixtures_on_device():
    lk = _lk()
    with open(os.path.join(GOLD, "quant_i8_worked.json")) as f:
        for case in json.load(f)["cases"]:
            if "v_ulps" in case:
                v = (np.array(case["v_ulps"], np.float64) * 2.0 ** -149).astype(np.float32)
            else:
                v = np.array(case["v"], np.float32)
            c, _ = lk.quantize_latent(to_dev(v[None]), "i8")
            assert c.cpu().numpy()[0].tolist() == case["codes"], case["name"]
    with open(os.path.join(GOLD, "quant_i4_worked.json")) as f:
        for case in json.load(f)["cases"]:
            v = np.array(case["v"], np.float32)
            c, s = lk.quantize_latent(to_dev(v[None]), "i4", case["group"])
            codes = O.unpack_i4(c.cpu().numpy()[0], len(v))
            assert codes.tolist() == case["codes"], case["name"]
            assert s.cpu().numpy()[0].astype(np.float64).tolist() == case["scales"], case["name"]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("m,k", [(1, 4096), (7, 11008), (33, 300), (5, 1)])
def test_quantize_rows_bit_exact(dtype, m, k):
    lk = _lk()
    g = torch.Generator().manual_seed(m * 1000 + k)
    x = (torch.randn(m, k, generator=g) * 3).to(dtype)
    q, s = lk.quantize_rows_i8(x.cuda())
    oq, os_ = O.quantize_rows_i8(x.float().numpy())
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_rmsnorm_quant_band(dtype):
    lk = _lk()
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(37, 4096, generator=g) * 2).to(dtype)
    q, s = lk.rmsnorm_quant_i8(x.cuda(), 1e-5)
    y32 = O.rmsnorm(x.float().numpy(), 1e-5).astype(np.float32)
    flips = check_codes_band(q.cpu().numpy(), s.cpu().numpy(), y32)
    assert flips <= 3


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_swiglu_quant_band(dtype):
    lk = _lk()
    g = torch.Generator().manual_seed(8)
    gate = (torch.randn(33, 11008, generator=g) * 3).to(dtype)
    up = torch.randn(33, 11008, generator=g).to(dtype)
    q, s = lk.swiglu_quant_i8(gate.cuda(), up.cuda())
    h32 = O.swiglu(gate.float().numpy(), up.float().numpy()).astype(np.float32)
    flips = check_codes_band(q.cpu().numpy(), s.cpu().numpy(), h32)
    assert flips <= 5
