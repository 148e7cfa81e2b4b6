"""Test helpers: oracle-built caches and comparison rules.

Comparison rules used by the GPU parity tests:
  * codes produced from identical float32 inputs: bit-exact;
  * codes whose float32 input was summed in a different order on the GPU
    (projection, RMSNorm, SwiGLU): equal, except a difference of exactly one
    where the oracle's ratio v/s lies within `band` of a rounding tie (k + 1/2)
    or where the row's scale itself differs by a few ulps;
  * float outputs: max |err| <= tol * RMS(oracle output) with tol 1e-5 for
    fp32 outputs and 1e-2 for bf16 outputs; a bf16 output additionally may
    carry its own storage rounding, at most half a bf16 ulp, i.e.
    2^-8 * |value| (assert_close_bf16).
  * float32 latents summed in a different order (length-E dot products):
    scales agree to a relative 1e-4 and codes may differ by one only within
    2e-3 (in code units) of a rounding tie.  For these inputs the fp32
    rounding of a length-E sum is about sqrt(E) * 2^-24 * sum|x a| / |v|,
    below 1e-4 relative for E <= 4096.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O


def oracle_codes_to_rows(codes, kind):
    """Logical code bytes of one (b, h): int8 codes -> uint8 view; int4 -> packed."""
    if kind == "i8":
        return np.asarray(codes, np.int8).view(np.uint8)
    return O.pack_i4(codes)


def build_caches(latents_k, latents_v, ranks_k, ranks_v, kind, group):
    """Quantise per-(b, h) latents with the oracle; return (oracle caches, rows/scales for the device)."""
    B = len(latents_k)
    ok, ov = O.LatentCache(B, ranks_k, kind, group), O.LatentCache(B, ranks_v, kind, group)
    rows_k, sc_k, rows_v, sc_v = [], [], [], []
    for b in range(B):
        qk = [(O.quantize_i8(v) if kind == "i8" else O.quantize_i4(v, min(group, r)))
              for v, r in zip(latents_k[b], ranks_k)]
        qv = [(O.quantize_i8(v) if kind == "i8" else O.quantize_i4(v, min(group, r)))
              for v, r in zip(latents_v[b], ranks_v)]
        ok.append(b, qk)
        ov.append(b, qv)
        rows_k.append([oracle_codes_to_rows(c, kind) for c, _ in qk])
        sc_k.append([s for _, s in qk])
        rows_v.append([oracle_codes_to_rows(c, kind) for c, _ in qv])
        sc_v.append([s for _, s in qv])
    return ok, ov, (rows_k, sc_k), (rows_v, sc_v)


def rms(x):
    x = np.asarray(x, np.float64)
    return float(np.sqrt(np.mean(x * x)))


def assert_close_rms(got, want, tol, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.max(np.abs(got - want)))
    scale = rms(want)
    assert err <= tol * scale, f"{what}: max|err| {err:.3e} > {tol:.0e} * RMS {scale:.3e}"
    return err / scale if scale else err


def assert_close_bf16(got, want, tol=1e-2, what="", ulps=0.5):
    """|got - want| <= tol * RMS(want) + ulps * 2^-7 |want|.

    2^-7 |v| bounds one bf16 ulp of v, so the default allows the output's own
    rounding (half an ulp); chained stages that re-store bf16 values pass ulps=1."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    scale = rms(want)
    err = np.abs(got - want)
    allowed = tol * scale + ulps * 2.0 ** -7 * np.abs(want)
    worst = int(np.argmax(err - allowed))
    assert np.all(err <= allowed), (f"{what}: |err| {err.flat[worst]:.3e} > {allowed.flat[worst]:.3e} "
                                    f"at value {want.flat[worst]:.3e} (RMS {scale:.3e})")
    return float(np.max(err)) / scale if scale else float(np.max(err))


def f32_ulp_diff(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


# Largest deviations the band rule has let through in this session (printed
# in the test summary so that the slack actually used is visible).
BAND_STATS = {"codes": 0, "flips": 0, "max_flip_tie_distance": 0.0, "max_scale_rel": 0.0,
              "max_scale_fp16_ulps": 0.0}


def check_codes_band(gpu_codes, gpu_scale, v32, kind="i8", group=32, band=2e-3, scale_rel=1e-4):
    """Compare device codes (unpacked, [n, r]) and scales against the oracle
    quantisation of the oracle's own float32 values v32 [n, r].

    Returns the number of codes that differ (each by exactly one, at a tie)."""
    v32 = np.asarray(v32, np.float32)
    if kind == "i8":
        oc, os_ = O.quantize_i8(v32)
        s_or = os_.astype(np.float64)[:, None]
        s_gpu = np.asarray(gpu_scale, np.float32)
        rel = np.abs(s_gpu.astype(np.float64) - os_) / np.maximum(os_.astype(np.float64), 1e-45)
        assert np.all(rel <= scale_rel), f"scale differs by {rel.max():.2e} relative"
        BAND_STATS["max_scale_rel"] = max(BAND_STATS["max_scale_rel"], float(rel.max(initial=0.0)))
        s_gpu_b = np.broadcast_to(s_gpu.astype(np.float64)[:, None], v32.shape)
    else:
        oc, os_ = O.quantize_i4(v32, group)
        idx = np.arange(v32.shape[1]) // group
        s_or = os_.astype(np.float64)[:, idx]
        s16_gpu = np.asarray(gpu_scale, np.float16)
        d = np.abs(s16_gpu.astype(np.float32).view(np.int32).astype(np.int64)
                   - os_.astype(np.float32).view(np.int32).astype(np.int64))
        # one fp16 ulp is 2^13 float32 ulps
        assert np.all(d <= 8192), "fp16 scale differs by more than one fp16 ulp"
        BAND_STATS["max_scale_fp16_ulps"] = max(BAND_STATS["max_scale_fp16_ulps"], float(d.max(initial=0)) / 8192)
        s_gpu_b = s16_gpu.astype(np.float64)[:, idx]
    gc = np.asarray(gpu_codes, np.int64)
    diff = gc - oc.astype(np.int64)
    bad = diff != 0
    BAND_STATS["codes"] += int(gc.size)
    if not bad.any():
        return 0
    assert np.all(np.abs(diff[bad]) == 1), "a code differs by more than one"
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = v32.astype(np.float64) / s_or
        ratio_gpu = v32.astype(np.float64) / s_gpu_b
    tie_dist = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5)
    near_tie = tie_dist <= band
    scale_moved = np.floor(ratio + 0.5) != np.floor(ratio_gpu + 0.5)
    ok = near_tie | scale_moved
    assert np.all(ok[bad]), f"{int(np.sum(bad & ~ok))} codes differ away from a rounding tie"
    BAND_STATS["flips"] += int(bad.sum())
    flip_d = tie_dist[bad & near_tie]
    if flip_d.size:
        BAND_STATS["max_flip_tie_distance"] = max(BAND_STATS["max_flip_tie_distance"], float(flip_d.max()))
    return int(bad.sum())


def to_dev(a, dtype=None, device="cuda"):
    t = torch.as_tensor(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)
