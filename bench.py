#!/usr/bin/env python3
"""Decode-step benchmark of the per-head latent-KV path on B200.

Default line: one autoregressive decode step of the LASER-style ragged-rank
workload across all of its layers (32 layers x 32 heads x H = 128, ranks
r_h in {8, 16, 32, 48, 64} per (layer, head), K and V drawn independently,
int8 latents, batch 8, 16384 cached tokens + the new one): per layer the new
token's latent projection + quantise + append and the latent flash-decode
attention, through lk_latent_decode_step.  The 10.7 GB working set lives in
HBM before timing and is far larger than L2.  Each step is timed with CUDA
events on the launching stream, the max over ranks is taken, and rank 0
prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 4]

--workload 1..3 time the single-layer appending workloads instead (L2
flushed before every step); --impl reference times the CPU oracle (float64,
K and V materialised) on the host cores, same workload and metric, on a
bounded sample of each step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s and latent-attn HBM GB/s (% of B200 peak) at 1 GPU"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.txt")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layer", action="store_true",
                    help="time one full W8A8 decoder-layer decode step (workload 5 shape); the latent cache "
                         "holds seeded random codes (no prefill)")
    ap.add_argument("--attn-only", action="store_true",
                    help="time the latent decode attention alone on one layer of the workload, "
                         "its cache filled with seeded random codes (no prefill)")
    ap.add_argument("--proj-only", action="store_true",
                    help="time the decode-step latent projection + quantise + append alone on one layer of the "
                         "workload (one new token per row; seq_len rewound outside the timed region)")
    ap.add_argument("--ffn-compare", action="store_true",
                    help="time the FFN input side (gate, up, SwiGLU, int8 requant) of the W8A8 layer shape with the "
                         "hybrid split on input channels (two hybrid linears + SwiGLU) and on output channels "
                         "(lk_ffn_gate_up_swiglu + requant)")
    ap.add_argument("--rope", action="store_true",
                    help="time the rotary-position decode (keys rebuilt on chip) against the absorbed latent decode "
                         "on one layer of workloads 2-4 (the same caches)")
    ap.add_argument("--all-layers", action="store_true",
                    help="kept for old command lines: multi-layer workloads always time every layer")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the extra single-layer B = 1 measurement in the default line")
    ap.add_argument("--dense-compare", action="store_true",
                    help="time one layer's latent attention against this library's dense bf16 flash-decoding "
                         "over materialised K/V and the naive rebuild-then-attend path, workloads 2-5")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- ranks

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cpu"):
    """Max of a float over all ranks (every rank takes this collective step)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks (NVML, read-only)

_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and throttle reasons every few ms while running (read-only NVML)."""

    def __init__(self, device_index, period_s=0.005, enabled=True):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        if not enabled:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= int(self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        reasons = [n for bit, n in _REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- workload state

class DecodeState:
    """Device state of the attention-layer decode workload (one layer)."""

    def __init__(self, w, device):
        import rank_latent_kv_lk_b200 as lk
        from rank_latent_kv_lk_b200 import synth
        self.lk, self.w = lk, w
        rk, rv = synth.ranks(w)
        self.rk, self.rv = rk[0], rv[0]
        A, BK, BV = synth.factors(w, 0, self.rk, self.rv)
        self.A, self.BK, self.BV = A.to(device), BK.to(device), BV.to(device)
        self.ck = lk.LatentCache(w.batch, self.rk, w.capacity, w.kind, w.group, device)
        self.cv = lk.LatentCache(w.batch, self.rv, w.capacity, w.kind, w.group, device, role="v")
        self.seq = torch.zeros(w.batch, dtype=torch.int32, device=device)
        x_ctx = synth.context_tokens(w, 0).to(device)
        lk.latent_project_append(self.ck, self.cv, x_ctx.reshape(-1, w.embed_dim), self.A, self.seq,
                                 [0] * w.batch)
        del x_ctx
        self.lens = w.context
        self.x_dec = synth.decode_tokens(w, 0).to(device)          # [steps, B, E]
        self.q = synth.queries(w, 0).to(device)                    # [steps, B, nh, H]
        self.out = torch.empty(w.batch, w.n_heads, w.head_dim, dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize()
        lk.device_status()

    def rewind_if_full(self):
        if self.lens >= self.w.context + self.w.steps:
            self.seq.fill_(self.w.context)
            self.lens = self.w.context

    def project(self, i, x=None):
        j = i % self.w.steps
        self.lk.latent_project_append(self.ck, self.cv, self.x_dec[j] if x is None else x, self.A, self.seq,
                                      [self.lens] * self.w.batch)
        self.lens += 1

    def step(self, i, x=None, q=None, out=None):
        """Append + attention through the decode step entry point (the attention
        launch overlaps the append)."""
        j = i % self.w.steps
        o = self.lk.latent_decode_step(self.ck, self.cv, self.x_dec[j] if x is None else x, self.A, self.seq,
                                       [self.lens] * self.w.batch, self.q[j] if q is None else q, self.BK,
                                       self.BV, out=self.out if out is None else out)
        self.lens += 1
        return o

    def attend(self, i, q=None, out=None):
        j = i % self.w.steps
        return self.lk.latent_decode_attn(self.ck, self.cv, self.q[j] if q is None else q, self.BK, self.BV,
                                          self.seq, self.lens, out=self.out if out is None else out)

    # algorithmic bytes (what the math must touch once)
    def attn_bytes(self, length):
        w = self.w
        rb = lambda r: r if w.kind == "i8" else r // 2
        sb = lambda r: 4 if w.kind == "i8" else 2 * (-(-r // min(w.group, r)))
        per_tok = sum(rb(r) + sb(r) for r in self.rk) + sum(rb(r) + sb(r) for r in self.rv)
        factors = (sum(self.rk) + sum(self.rv)) * w.head_dim * self.BK.element_size()
        qo = 2 * w.batch * w.n_heads * w.head_dim * 2
        return w.batch * length * per_tok + factors + qo

    def proj_bytes(self):
        w = self.w
        rb = lambda r: r if w.kind == "i8" else r // 2
        codes = w.batch * (sum(rb(r) for r in self.rk) + sum(rb(r) for r in self.rv))
        return self.A.numel() * self.A.element_size() + w.batch * w.embed_dim * 2 + codes


# sources each profiled kernel is built from (its traffic figure stays valid
# while these are unchanged)
KERNEL_SOURCES = {
    "decode_attn_kernel": ["lk_decode.cu", "lk_common.cuh", "lk_internal.h"],
    "proj_cluster_kernel": ["lk_project.cu", "lk_common.cuh", "lk_quant.cuh", "lk_internal.h"],
    "proj_mma_kernel": ["lk_project.cu", "lk_common.cuh", "lk_quant.cuh", "lk_internal.h"],
}


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rank_latent_kv_lk_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(ROOT, "include", "lk.h"), "rb") as f:
        h.update(b"lk.h" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's sources have not changed since."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            for line in f:
                parts = line.split()
                if not parts or parts[0].startswith("#"):
                    continue
                if parts[0] == f"{kernel}@{workload}" and parts[2] == kernel_source_hash(kernel):
                    return int(parts[1])
    except OSError:
        pass
    return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_session(w):
    """Oracle state of a single-layer appending workload after its (untimed)
    context prefill; returns a step function (one decode step of the workload)."""
    import oracle as O
    from rank_latent_kv_lk_b200 import synth
    rk, rv = synth.ranks(w)
    rk, rv = rk[0], rv[0]
    A, BK, BV = synth.factors(w, 0, rk, rv)
    A64 = synth.as_numpy(A).T.astype(np.float64)
    BK, BV = synth.as_numpy(BK).astype(np.float64), synth.as_numpy(BV).astype(np.float64)
    offk, offv = np.cumsum([0] + rk), np.cumsum([0] + rv)
    BKh = [BK[offk[h]:offk[h + 1]] for h in range(len(rk))]
    BVh = [BV[offv[h]:offv[h + 1]] for h in range(len(rv))]
    ck, cv = O.LatentCache(w.batch, rk, w.kind, w.group), O.LatentCache(w.batch, rv, w.kind, w.group)
    nk = sum(rk)
    x_ctx = synth.as_numpy(synth.context_tokens(w, 0))
    for b in range(w.batch):
        v = O.latent_project_float(x_ctx[b], A64)
        ck.append(b, O.quantize_latents(v[:, :nk], rk, w.kind, w.group))
        cv.append(b, O.quantize_latents(v[:, nk:], rv, w.kind, w.group))
    x_dec = synth.as_numpy(synth.decode_tokens(w, 0))
    q = synth.as_numpy(synth.queries(w, 0))
    scale = 1.0 / math.sqrt(w.head_dim)

    def step(i):
        j = i % w.steps
        v = O.latent_project_float(x_dec[j], A64)
        for b in range(w.batch):
            ck.append(b, O.quantize_latents(v[b:b + 1, :nk], rk, w.kind, w.group))
            cv.append(b, O.quantize_latents(v[b:b + 1, nk:], rv, w.kind, w.group))
        return O.latent_attention(q[j], ck, cv, BKh, BVh, scale)

    return step


class OracleLayerSample:
    """Bounded samples of one decode step of a multi-layer workload for the CPU
    oracle.  A full step (every layer, every (b, h) over T tokens, K and V
    materialised in float64) takes the oracle many minutes, so a sample is one
    (layer, b, h) unit: that layer's projection of the new tokens (its share
    per unit), then the unit's quantise + append and its attention over the
    cache, whose T - 1 context codes and scales are seeded random draws like
    the device bench's.  A step's time is a unit's time times the units of
    all layers."""

    def __init__(self, w):
        import oracle as O
        from rank_latent_kv_lk_b200 import synth
        self.O, self.w = O, w
        self.rks, self.rvs = synth.ranks(w)
        self.T = w.context + 1
        self.units = w.n_layers * w.batch * w.n_heads
        self._synth = synth
        self._layer = None

    def _load_layer(self, l):
        if self._layer is not None and self._layer[0] == l:
            return self._layer
        w, synth = self.w, self._synth
        A, BK, BV = synth.factors(w, l, self.rks[l], self.rvs[l])
        A64 = synth.as_numpy(A).T.astype(np.float64)
        BK, BV = synth.as_numpy(BK).astype(np.float64), synth.as_numpy(BV).astype(np.float64)
        x = synth.as_numpy(synth.decode_tokens(w, l)[0])
        q = synth.as_numpy(synth.queries(w, l)[0])
        self._layer = (l, A64, BK, BV, x, q)
        return self._layer

    def unit(self, i):
        """Oracle work of unit i (cycling over (layer, b, h)).  Returns the
        seconds the oracle took; drawing the unit's random context codes is
        not timed."""
        O, w = self.O, self.w
        u = i % self.units
        l, rest = divmod(u, w.batch * w.n_heads)
        b, h = divmod(rest, w.n_heads)
        l, A64, BK, BV, x, q = self._load_layer(l)
        rk, rv = self.rks[l], self.rvs[l]
        nk = sum(rk)
        rng = np.random.default_rng(1000003 * (l + 1) + 1009 * b + h)
        ck, cv = O.LatentCache(1, [rk[h]], w.kind, w.group), O.LatentCache(1, [rv[h]], w.kind, w.group)
        ctx = []
        for r in (rk[h], rv[h]):
            codes = rng.integers(-127, 128, (self.T - 1, r), dtype=np.int64).astype(np.int8)
            scales = (rng.random(self.T - 1) * 0.02 + 0.01).astype(np.float32)
            ctx.append((codes, scales))
        t0 = time.perf_counter()
        ck.append(0, [ctx[0]])
        cv.append(0, [ctx[1]])
        # this unit's share of the layer's projection: the new token's latent of head h (K and V)
        ok, ov = sum(rk[:h]), nk + sum(rv[:h])
        vk = O.latent_project_float(x[b:b + 1], A64[:, ok:ok + rk[h]])
        vv = O.latent_project_float(x[b:b + 1], A64[:, ov:ov + rv[h]])
        ck.append(0, O.quantize_latents(vk, [rk[h]], w.kind, w.group))
        cv.append(0, O.quantize_latents(vv, [rv[h]], w.kind, w.group))
        offk, offv = sum(rk[:h]), sum(rv[:h])
        O.latent_attention(q[b:b + 1, h:h + 1], ck, cv, [BK[offk:offk + rk[h]]],
                           [BV[offv:offv + rv[h]]], 1.0 / math.sqrt(w.head_dim))
        return time.perf_counter() - t0

    def sample_text(self, n):
        w = self.w
        return (f"{n} (layer, b, h) units of the {w.n_layers}-layer step, each: its share of the layer's "
                f"projection of the new token, quantise + append, and float64 attention with K and V "
                f"materialised over {self.T} tokens (drawing the unit's random context codes untimed); "
                f"step time = mean unit time x {self.units} units")


def _timed_units(sample, budget_s, max_units=None):
    """Oracle seconds over units until about budget_s of wall time has passed."""
    t0 = time.perf_counter()
    n, dt = 0, 0.0
    while True:
        dt += sample.unit(n)
        n += 1
        if time.perf_counter() - t0 >= budget_s or (max_units and n >= max_units):
            return n, dt


def cpu_baseline(w, budget_s=12.0):
    """The oracle on the host cores: all the cores this process may use, and one thread."""
    cores = host_cores()
    try:
        import threadpoolctl
    except ImportError:
        threadpoolctl = None
    if w.n_layers > 1:
        sample = OracleLayerSample(w)
        sample.unit(0)  # warm-up (first layer load)
        n, dt = _timed_units(sample, budget_s)
        value = w.batch / (dt / n * sample.units)
        single = None
        if threadpoolctl is not None:
            with threadpoolctl.threadpool_limits(1):
                n1, dt1 = _timed_units(sample, budget_s / 2)
            single = w.batch / (dt1 / n1 * sample.units)
        return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                "single_thread_value": single, "sample": sample.sample_text(n)}
    step = oracle_session(w)
    t0 = time.perf_counter()
    step(0)
    t1 = time.perf_counter() - t0
    n = int(max(1, min(w.steps - 1, budget_s / max(t1, 1e-6))))
    t0 = time.perf_counter()
    for i in range(1, n + 1):
        step(i)
    dt = time.perf_counter() - t0
    single = None
    if threadpoolctl is not None:
        with threadpoolctl.threadpool_limits(1):
            t0 = time.perf_counter()
            m = max(1, n // 2)
            for i in range(n + 1, n + 1 + m):
                step(i)
            single = w.batch * m / (time.perf_counter() - t0)
    return {"value": w.batch * n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "single_thread_value": single,
            "sample": f"{n} decode steps of the workload after its context prefill (prefill untimed; "
                      f"float64, K and V materialised)"}


# ---------------------------------------------------------------- arms

def workload_dtype(w):
    codes = "int8" if w.kind == "i8" else "int4"
    acts = {"f32": "f32", "bf16": "bf16", "i8": "int8"}[w.act]
    return f"{codes} latents, {acts} activations and factors, f32 accumulate"


def workload_data(w):
    if w.n_layers > 1:
        return ("synthetic (seeded): random int8 latent codes and positive scales in every cache (no prefill), "
                "factors A ~ N(0, 1/E) and B ~ N(0, 1/r) in bf16, x and q ~ N(0, 1) per layer")
    extra = f", first {w.image_tokens} context tokens sigma {w.image_sigma}" if w.image_tokens else ""
    if w.outlier_frac:
        extra += f", {w.outlier_frac:.0%} of x channels x{w.outlier_scale:g}"
    return f"synthetic (seeded): x ~ N(0, 1){extra}, prefilled through the library; q ~ N(0, 1) per step"


def run_reference(args):
    """The CPU oracle as the reference arm: same workload, metric and unit; each
    step is a bounded sample of a decode step (a unit of it for multi-layer
    workloads), its time scaled to the whole step."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    w = WORKLOADS[args.workload]
    if w.n_layers > 1:
        sample = OracleLayerSample(w)
        for i in range(args.warmup):
            sample.unit(i)
        dt = sum(sample.unit(i) for i in range(args.warmup, args.warmup + args.steps))
        step_s = dt / args.steps * sample.units
        value = w.batch / step_s
        text = sample.sample_text(args.steps) + f", after {args.warmup} warm-up units"
        config = {"workload": w.name, "layers": w.n_layers, "batch": w.batch, "tokens": w.context + 1}
    else:
        step = oracle_session(w)
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        for i in range(args.warmup, args.warmup + args.steps):
            step(i)
        dt = time.perf_counter() - t0
        step_s = dt / args.steps
        value = w.batch / step_s
        text = (f"{args.steps} timed oracle decode steps after {args.warmup} warm-up steps and an untimed "
                "context prefill")
        config = {"workload": w.name, "batch": w.batch, "context": w.context}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": workload_data(w), "config": config,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
                             "sample": text},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    w = WORKLOADS[args.workload]
    if w.n_layers > 1:
        return run_multilayer(args, w)
    return run_single(args, w)


class MultiLayerState:
    """Device state of a multi-layer workload: per layer the K and V latent
    caches (seeded random codes and positive scales: their contents do not
    change the work), the factors, the new token x and the query q."""

    def __init__(self, w, device):
        import rank_latent_kv_lk_b200 as lk
        from rank_latent_kv_lk_b200 import synth
        self.lk, self.w = lk, w
        self.rks, self.rvs = synth.ranks(w)
        L = w.n_layers
        g = torch.Generator(device=device)
        g.manual_seed(synth.seed_for(w, synth.CONTEXT))
        self.layers = []
        for l in range(L):
            A, BK, BV = synth.factors(w, l, self.rks[l], self.rvs[l])
            ck = lk.LatentCache(w.batch, self.rks[l], w.capacity, w.kind, w.group, device)
            cv = lk.LatentCache(w.batch, self.rvs[l], w.capacity, w.kind, w.group, device, role="v")
            for c in (ck, cv):
                c.codes.copy_(torch.randint(0, 256, c.codes.shape, dtype=torch.uint8, device=device, generator=g))
                sc = torch.rand(c.scales.shape, device=device, generator=g) * 0.02 + 0.01
                c.scales.copy_(sc.to(c.scales.dtype))
            self.layers.append((ck, cv, A.to(device), BK.to(device), BV.to(device)))
        self.x = torch.stack([synth.decode_tokens(w, l)[0] for l in range(L)]).to(device)   # [L, B, E]
        self.q = torch.stack([synth.queries(w, l)[0] for l in range(L)]).to(device)         # [L, B, nh, H]
        self.out = torch.empty(L, w.batch, w.n_heads, w.head_dim, dtype=self.q.dtype, device=device)
        self.seq = torch.full((L, w.batch), w.context, dtype=torch.int32, device=device)
        self.lens0 = [w.context] * w.batch
        torch.cuda.synchronize()

    def reset(self):
        self.seq.fill_(self.w.context)

    def step(self, x=None, q=None, out=None):
        x = self.x if x is None else x
        q = self.q if q is None else q
        out = self.out if out is None else out
        for l, (ck, cv, A, BK, BV) in enumerate(self.layers):
            self.lk.latent_decode_step(ck, cv, x[l], A, self.seq[l], self.lens0, q[l], BK, BV, out=out[l])

    def attn_bytes(self, l):
        """Algorithmic bytes of one attention launch of layer l (cache of T tokens, factors, q, out)."""
        w = self.w
        T = w.context + 1
        rb = lambda r: r if w.kind == "i8" else r // 2
        sb = lambda r: 4 if w.kind == "i8" else 2 * (-(-r // min(w.group, r)))
        per_tok = sum(rb(r) + sb(r) for r in self.rks[l]) + sum(rb(r) + sb(r) for r in self.rvs[l])
        factors = (sum(self.rks[l]) + sum(self.rvs[l])) * w.head_dim * 2
        return w.batch * T * per_tok + factors + 2 * w.batch * w.n_heads * w.head_dim * 2

    def proj_bytes(self, l):
        w = self.w
        rb = lambda r: r if w.kind == "i8" else r // 2
        n_tot = sum(self.rks[l]) + sum(self.rvs[l])
        codes = w.batch * (sum(rb(r) for r in self.rks[l]) + sum(rb(r) for r in self.rvs[l]))
        return n_tot * w.embed_dim * 2 + w.batch * w.embed_dim * 2 + codes


def run_multilayer(args, w):
    """The headline: one decode step across every layer of the workload."""
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    st = MultiLayerState(w, device)
    lk = st.lk
    stream = torch.cuda.current_stream()
    L = w.n_layers
    for _ in range(max(3, args.warmup)):
        st.step()
        st.reset()
    torch.cuda.synchronize()
    lk.device_status()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e8))  # let the host queue run ahead of the device
    n0 = lk.kernel_launches()
    with ClockSampler(local) as clocks:
        for i in range(K):
            st.reset()
            ev[i][0].record(stream)
            st.step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    launches = lk.kernel_launches() - n0
    barrier(world)
    lk.device_status()
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    value = w.batch * K * world / (total_ms / 1e3)

    # per-kernel durations: a second pass with events between the two kernels
    # of every layer (for the roofline; the events stop the overlap of the two)
    KP = min(K, 10)
    kev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(L)] for _ in range(KP)]
    torch.cuda.synchronize()
    torch.cuda._sleep(int(1e8))
    for i in range(KP):
        st.reset()
        for l, (ck, cv, A, BK, BV) in enumerate(st.layers):
            kev[i][l][0].record(stream)
            lk.latent_project_append(ck, cv, st.x[l], A, st.seq[l], st.lens0)
            kev[i][l][1].record(stream)
            lk.latent_decode_attn(ck, cv, st.q[l], BK, BV, st.seq[l], w.context + 1, out=st.out[l])
            kev[i][l][2].record(stream)
    torch.cuda.synchronize()
    attn_s = sum(kev[i][l][1].elapsed_time(kev[i][l][2]) for i in range(KP) for l in range(L)) / 1e3
    proj_s = sum(kev[i][l][0].elapsed_time(kev[i][l][1]) for i in range(KP) for l in range(L)) / 1e3
    attn_bytes = KP * sum(st.attn_bytes(l) for l in range(L))
    proj_bytes = KP * sum(st.proj_bytes(l) for l in range(L))
    attn_gbs = attn_bytes / attn_s / 1e9
    proj_gbs = proj_bytes / proj_s / 1e9

    # e2e: every layer's x and q copied host -> device from pinned memory and
    # every layer's output copied back, inside the timed region
    e2e = None
    if not args.no_e2e:
        nx = st.x.numel() * st.x.element_size()
        nq = st.q.numel() * st.q.element_size()
        hbuf = torch.empty(nx + nq, dtype=torch.uint8).pin_memory()
        hbuf[:nx].copy_(st.x.reshape(-1).view(torch.uint8).cpu())
        hbuf[nx:].copy_(st.q.reshape(-1).view(torch.uint8).cpu())
        dbuf = torch.empty(nx + nq, dtype=torch.uint8, device=device)
        xd = dbuf[:nx].view(st.x.dtype).view(st.x.shape)
        qd = dbuf[nx:].view(st.q.dtype).view(st.q.shape)
        oh = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
        e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize()
        torch.cuda._sleep(int(1e8))
        for i in range(K):
            st.reset()
            e_ev[i][0].record(stream)
            dbuf.copy_(hbuf, non_blocking=True)
            st.step(x=xd, q=qd)
            oh.copy_(st.out, non_blocking=True)
            e_ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e_ev), world, device)
        e2e = {"value": w.batch * K * world / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": nx + nq,
               "d2h_bytes_per_step": oh.numel() * oh.element_size(),
               "path": "rank_latent_kv_lk_b200.latent_decode_step per layer (C ABI), inputs from pinned host "
                       "memory, outputs back to pinned host memory"}
    extra = None
    if not args.no_extra:
        from rank_latent_kv_lk_b200.configs import WORKLOADS
        del st
        torch.cuda.empty_cache()
        extra = measure_single(args, WORKLOADS[2], device, world, clocks_too=False, K=max(K, 128))

    if rank != 0:
        _finish(world)
        return 0
    hbm, peak_kind = peaks()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": workload_dtype(w), "data": workload_data(w),
        "config": {"workload": w.name, "layers": L, "batch": w.batch, "tokens": w.context + 1,
                   "l2": "not flushed: the 10.7 GB working set is far larger than L2 (126 MB)",
                   "timing": "CUDA events at step boundaries on the launching stream; max over ranks; "
                             "per-kernel times from a second pass with events between the kernels",
                   "parallelism": f"replicas x{world} (independent decode problems, no collective)"},
        "roofline": {"kernel": "decode_attn_kernel", "bound": "hbm", "achieved": attn_gbs, "peak": hbm,
                     "unit": "GB/s", "frac": attn_gbs / hbm, "peak_kind": peak_kind,
                     "frac_of_8tbs": attn_gbs / 8000.0,
                     "algorithmic_bytes_per_launch": attn_bytes / (KP * L),
                     "us_per_launch": attn_s / (KP * L) * 1e6,
                     "traffic": profiled_traffic("decode_attn_kernel", w.key)},
        "latent_project": {"achieved_gbs": proj_gbs, "us_per_call": proj_s / (KP * L) * 1e6,
                           "algorithmic_bytes_per_call": proj_bytes / (KP * L)},
        "step_algorithmic_gbs": (attn_bytes + proj_bytes) / KP / (total_ms / K / 1e3) / 1e9,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if e2e:
        line["e2e"] = e2e
    if extra:
        line["llava7b_b1_step"] = extra
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    _finish(world)
    return 0


def measure_single(args, w, device, world, clocks_too=True, K=None):
    """Appending decode steps of a single-layer workload (L2 flushed before
    every step); returns the measurements as a dict."""
    st = DecodeState(w, device)
    lk = st.lk
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for i in range(max(3, args.warmup)):
        st.rewind_if_full()
        st.step(i)
    torch.cuda.synchronize()
    K = K or args.steps
    # timed region: events at step boundaries only (an event between the two
    # kernels would stop the attention launch from overlapping the projection)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(1e8))
    n0 = lk.kernel_launches()
    with ClockSampler(device.index, enabled=clocks_too) as clocks:
        for i in range(K):
            st.rewind_if_full()
            flush.fill_(1)
            ev[i][0].record(stream)
            st.step(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    launches = lk.kernel_launches() - n0
    barrier(world)
    lk.device_status()
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    klens = []
    torch.cuda.synchronize()
    torch.cuda._sleep(int(1e8))
    for i in range(K):
        st.rewind_if_full()
        flush.fill_(1)
        kev[i][0].record(stream)
        st.project(i)
        kev[i][1].record(stream)
        st.attend(i)
        kev[i][2].record(stream)
        klens.append(st.lens)
    torch.cuda.synchronize()
    proj_s = statistics.mean(kev[i][0].elapsed_time(kev[i][1]) for i in range(K)) / 1e3
    attn_s = statistics.mean(kev[i][1].elapsed_time(kev[i][2]) for i in range(K)) / 1e3
    attn_bytes = statistics.mean(st.attn_bytes(n) for n in klens)
    e2e = None
    if not args.no_e2e:
        xs, qs = st.x_dec[0], st.q[0]
        nx = xs.numel() * xs.element_size()
        nq = qs.numel() * qs.element_size()
        hbuf = torch.empty(w.steps, nx + nq, dtype=torch.uint8).pin_memory()
        hbuf[:, :nx].copy_(st.x_dec.reshape(w.steps, -1).view(torch.uint8).cpu())
        hbuf[:, nx:].copy_(st.q.reshape(w.steps, -1).view(torch.uint8).cpu())
        oh = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
        dbuf = torch.empty(nx + nq, dtype=torch.uint8, device=device)
        xd = dbuf[:nx].view(xs.dtype).view(xs.shape)
        qd = dbuf[nx:].view(qs.dtype).view(qs.shape)
        e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize()
        torch.cuda._sleep(int(1e8))
        for i in range(K):
            j = i % w.steps
            st.rewind_if_full()
            flush.fill_(1)
            e_ev[i][0].record(stream)
            dbuf.copy_(hbuf[j], non_blocking=True)
            st.step(i, x=xd, q=qd)
            oh.copy_(st.out, non_blocking=True)
            e_ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e_ev), world, device)
        e2e = {"value": w.batch * K * world / (e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": nx + nq,
               "d2h_bytes_per_step": oh.numel() * oh.element_size()}
    res = {"workload": w.name, "value": w.batch * K * world / (total_ms / 1e3), "unit": UNIT, "steps": K,
           "ms_per_step": total_ms / K, "l2": "flushed before every step (256 MiB write, untimed)",
           "gpu_launches": launches,
           "attn_us_per_launch": attn_s * 1e6, "attn_gbs": attn_bytes / attn_s / 1e9,
           "attn_algorithmic_bytes_per_launch": attn_bytes,
           "proj_us_per_call": proj_s * 1e6, "proj_gbs": st.proj_bytes() / proj_s / 1e9,
           "proj_algorithmic_bytes_per_call": st.proj_bytes()}
    if e2e:
        res["e2e"] = e2e
    if clocks_too:
        res["clocks"] = clocks.summary()
    del st
    torch.cuda.empty_cache()
    return res


def run_single(args, w):
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    r = measure_single(args, w, device, world)
    if rank != 0:
        _finish(world)
        return 0
    hbm, peak_kind = peaks()
    dominant = "decode_attn_kernel" if r["attn_us_per_launch"] >= r["proj_us_per_call"] else (
        "proj_mma_kernel" if w.act == "bf16" else "proj_cluster_kernel")
    ach = r["attn_gbs"] if dominant == "decode_attn_kernel" else r["proj_gbs"]
    line = {
        "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": r["steps"],
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": workload_dtype(w), "data": workload_data(w),
        "config": {"workload": w.name, "batch": w.batch, "context": w.context, "decode_steps": w.steps,
                   "l2": r["l2"],
                   "timing": "CUDA events at step boundaries on the launching stream; max over ranks; "
                             "per-kernel times from a second pass of the same steps with an event between "
                             "the kernels",
                   "parallelism": f"replicas x{world} (independent decode problems, no collective)"},
        "roofline": {"kernel": dominant, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s",
                     "frac": ach / hbm, "peak_kind": peak_kind, "frac_of_8tbs": ach / 8000.0,
                     "traffic": profiled_traffic(dominant, w.key)},
        "latent_attn": {"achieved_gbs": r["attn_gbs"], "us_per_launch": r["attn_us_per_launch"],
                        "algorithmic_bytes_per_launch": r["attn_algorithmic_bytes_per_launch"]},
        "latent_project": {"achieved_gbs": r["proj_gbs"], "us_per_call": r["proj_us_per_call"],
                           "algorithmic_bytes_per_call": r["proj_algorithmic_bytes_per_call"]},
        "gpu_launches": r["gpu_launches"], "clocks": r.get("clocks"),
    }
    if "e2e" in r:
        line["e2e"] = r["e2e"]
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    _finish(world)
    return 0


def run_proj_only(args):
    """The decode-step latent projection + quantise + append alone on one layer
    of a workload (one new token per batch row), L2 flushed before every call."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    import rank_latent_kv_lk_b200 as lk
    from rank_latent_kv_lk_b200 import synth
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    w = WORKLOADS[args.workload]
    rk, rv = synth.ranks(w)
    rk, rv = rk[0], rv[0]
    A, _, _ = synth.factors(w, 0, rk, rv)
    A = A.to(device)
    cap = 64
    ck = lk.LatentCache(w.batch, rk, cap, w.kind, w.group, device)
    cv = lk.LatentCache(w.batch, rv, cap, w.kind, w.group, device, role="v")
    seq = torch.zeros(w.batch, dtype=torch.int32, device=device)
    x = synth.decode_tokens(w, 0)[0].to(device)
    if x.dtype != A.dtype:
        x = x.to(A.dtype)
    x_scale = a_scale = None
    if w.act == "i8":
        raise SystemExit("--proj-only covers the float workloads (1-4)")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    hl = [0] * w.batch
    for _ in range(max(3, args.warmup)):
        seq.zero_()
        lk.latent_project_append(ck, cv, x, A, seq, hl, x_scale, a_scale)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(1e8))
    with ClockSampler(local) as clocks:
        for i in range(K):
            seq.zero_()
            flush.fill_(1)
            ev[i][0].record(stream)
            lk.latent_project_append(ck, cv, x, A, seq, hl, x_scale, a_scale)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    lk.device_status()
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    us = total_ms / K * 1e3
    esz = A.element_size()
    rb = lambda r: r if w.kind == "i8" else r // 2
    sb = lambda r: 4 if w.kind == "i8" else 2 * (-(-r // min(w.group, r)))
    new_bytes = w.batch * (sum(rb(r) + sb(r) for r in rk) + sum(rb(r) + sb(r) for r in rv))
    nbytes = A.numel() * esz + x.numel() * x.element_size() + new_bytes
    gbs = nbytes / (us * 1e-6) / 1e9
    hbm, peak_kind = peaks()
    kernel = "proj_mma_kernel" if w.act == "bf16" else "proj_cluster_kernel"
    if rank == 0:
        print(json.dumps({
            "mode": "proj-only", "metric": "latent-projection HBM GB/s", "value": gbs * world, "unit": "GB/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "us_per_call": us, "higher_is_better": True,
            "scaling": "weak", "dtype": w.act,
            "data": "synthetic (seeded: the workload's decode tokens and factors)",
            "config": {"workload": w.name, "layer": 0, "batch": w.batch, "n_tot": int(A.shape[0]),
                       "embed_dim": w.embed_dim, "l2": "flushed before every call (256 MiB write, untimed)"},
            "algorithmic_bytes_per_call": nbytes,
            "roofline": {"kernel": kernel, "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "peak_kind": peak_kind,
                         "traffic": profiled_traffic(kernel, f"{w.key}-proj")},
            "clocks": clocks.summary(),
        }))
    if world > 1:
        torch.distributed.destroy_process_group()


def run_ffn_compare(args):
    """FFN input side at the W8A8 layer shape, the two channel splits side by side."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import rank_latent_kv_lk_b200 as lk
    from rank_latent_kv_lk_b200 import synth
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    from rank_latent_kv_lk_b200.layer import hybrid_weight
    w = WORKLOADS[5]
    rk, rv = synth.ranks(w)
    lw = synth.layer_weights_w8a8(w, rk[0], rv[0])
    gate_in = hybrid_weight(lw["gate"], w.embed_dim, w.ffn_inter, device)
    up_in = hybrid_weight(lw["up"], w.embed_dim, w.ffn_inter, device)
    d = synth.ffn_outsplit_weights(w)
    ffn = lk.OutsplitFfn(d, device)
    g = torch.Generator().manual_seed(5)
    xq = torch.clamp(torch.round(torch.randn(w.batch, w.embed_dim, generator=g) * 40), -127, 127).to(torch.int8)
    xq = xq.to(device)
    sx = (torch.rand(w.batch, generator=g) * 0.01 + 0.002).to(device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def split_in():
        gg = lk.lowrank_linear(gate_in, xq, sx)
        uu = lk.lowrank_linear(up_in, xq, sx)
        return lk.swiglu_quant_i8(gg, uu)

    def split_out():
        return lk.quantize_rows_i8(ffn(xq, sx))

    def timed(fn, K):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        l0 = lk.kernel_launches()
        for i in range(K):
            flush.fill_(1)
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        return sum(e[0].elapsed_time(e[1]) for e in ev) / K * 1e3, (lk.kernel_launches() - l0) / K

    K = args.steps
    us_in, n_in = timed(split_in, K)
    us_out, n_out = timed(split_out, K)
    nbytes = lambda dd: sum(v.numel() * v.element_size() for k in ("gate", "up") for v in dd[k].values())
    b_in = sum(t.numel() * t.element_size() for name in ("gate", "up")
               for t in (lw[name]["W_D"], lw[name]["U"], lw[name]["V"]))
    b_out = nbytes(d)
    hbm, peak_kind = peaks()
    if rank == 0:
        print(json.dumps({
            "mode": "ffn-compare", "workload": w.name, "batch": w.batch, "hidden": w.ffn_inter,
            "l2": "flushed before every call (256 MiB write, untimed)",
            "input_split": {"us": us_in, "launches": n_in, "weight_bytes": b_in, "gbs": b_in / us_in / 1e3},
            "output_split_fused": {"us": us_out, "launches": n_out, "weight_bytes": b_out,
                                   "gbs": b_out / us_out / 1e3},
            "peak_gbs": hbm, "peak_kind": peak_kind,
        }))


def run_attn_only(args):
    """Latent decode attention alone on one layer of a workload (throughput of
    the cache stream at the large shapes).  The cache holds seeded random codes
    and positive scales; q and the factors follow the workload's recipe."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    import rank_latent_kv_lk_b200 as lk
    from rank_latent_kv_lk_b200 import synth
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    w = WORKLOADS[args.workload]
    rk, rv = synth.ranks(w)
    rk, rv = rk[0], rv[0]
    _, BK, BV = synth.factors(w, 0, rk, rv)
    BK, BV = BK.to(device), BV.to(device)
    T = w.context + 1
    g = torch.Generator(device=device)
    g.manual_seed(synth.seed_for(w, synth.CONTEXT))
    caches = []
    for ranks in (rk, rv):
        c = lk.LatentCache(w.batch, ranks, w.capacity, w.kind, w.group, device, role="k" if not caches else "v")
        c.codes.copy_(torch.randint(0, 256, c.codes.shape, dtype=torch.uint8, device=device, generator=g))
        sc = torch.rand(c.scales.shape, device=device, generator=g) * 0.02 + 0.01
        c.scales.copy_(sc.to(c.scales.dtype))
        caches.append(c)
    ck, cv = caches
    q = synth.queries(w, 0)[0].to(device)
    seq = torch.full((w.batch,), T, dtype=torch.int32, device=device)
    out = torch.empty(w.batch, w.n_heads, w.head_dim, dtype=torch.bfloat16, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    for _ in range(max(3, args.warmup)):
        lk.latent_decode_attn(ck, cv, q, BK, BV, seq, T, out=out)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(1e8))
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush.fill_(1)
            ev[i][0].record(stream)
            lk.latent_decode_attn(ck, cv, q, BK, BV, seq, T, out=out)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    lk.device_status()
    ms = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(ms), world, device)
    rb = lambda r: r if w.kind == "i8" else r // 2
    sb = lambda r: 4 if w.kind == "i8" else 2 * (-(-r // min(w.group, r)))
    per_tok = sum(rb(r) + sb(r) for r in rk) + sum(rb(r) + sb(r) for r in rv)
    nbytes = w.batch * T * per_tok + (sum(rk) + sum(rv)) * w.head_dim * 2 + 2 * w.batch * w.n_heads * w.head_dim * 2
    us = total_ms / K * 1e3
    gbs = nbytes / (us * 1e-6) / 1e9
    hbm, peak_kind = peaks()
    if rank == 0:
        print(json.dumps({
            "mode": "attn-only", "metric": "latent-attn HBM GB/s", "value": gbs * world, "unit": "GB/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "us_per_launch": us, "higher_is_better": True,
            "scaling": "weak", "dtype": "int8/f32" if w.kind == "i8" else "int4/f32",
            "data": "synthetic (seeded random latent codes and scales; shapes of the workload)",
            "config": {"workload": w.name, "layer": 0, "batch": w.batch, "tokens": T,
                       "l2": "flushed before every launch (256 MiB write, untimed)"},
            "algorithmic_bytes_per_launch": nbytes,
            "roofline": {"kernel": "latent_decode_attn", "bound": "hbm", "achieved": gbs, "peak": hbm,
                         "unit": "GB/s", "frac": gbs / hbm, "peak_kind": peak_kind,
                         "frac_of_8tbs": gbs / 8000.0,
                         "traffic": profiled_traffic("decode_attn_kernel", f"{w.key}-attn")},
            "gpu_launches": K, "clocks": clocks.summary()}), flush=True)
    _finish(world)
    return 0


def run_layer(args):
    """One W8A8 decoder-layer decode step (RMSNorm+quant, W_Q, latent append,
    latent attention, quant, W_O + residual, RMSNorm+quant, hybrid gate/up,
    SwiGLU+quant, hybrid down + residual), all through the C ABI."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    import rank_latent_kv_lk_b200 as lk
    from rank_latent_kv_lk_b200 import synth
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    from rank_latent_kv_lk_b200.layer import W8A8DecoderLayer
    w = WORKLOADS[5]
    rk, rv = synth.ranks(w)
    rk, rv = rk[0], rv[0]
    wts = synth.layer_weights_w8a8(w, rk, rv)
    layer = W8A8DecoderLayer(wts, w.n_heads, w.head_dim, rk, rv, w.batch, w.capacity, w.ffn_inter, device)
    g = torch.Generator(device=device)
    g.manual_seed(synth.seed_for(w, synth.CONTEXT))
    for c in (layer.cache_k, layer.cache_v):
        c.codes.copy_(torch.randint(0, 256, c.codes.shape, dtype=torch.uint8, device=device, generator=g))
        c.scales.copy_(torch.rand(c.scales.shape, device=device, generator=g) * 0.02 + 0.01)
    xs = synth.decode_tokens(w, 0).to(device)  # [steps, B, E] bf16
    seq = torch.full((w.batch,), w.context, dtype=torch.int32, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    lens = [w.context] * w.batch
    for i in range(max(3, args.warmup)):
        layer.step(xs[i % w.steps], seq, lens)
        seq.fill_(w.context)
        lens = [w.context] * w.batch
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e8))
    with ClockSampler(local) as clocks:
        for i in range(K):
            if i % w.steps == 0 and i:
                seq.fill_(w.context)
                lens = [w.context] * w.batch
            flush.fill_(1)
            ev[i][0].record(stream)
            layer.step(xs[i % w.steps], seq, lens)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    lk.device_status()
    total_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), world, device)
    us_eager = total_ms / K * 1e3

    # the same step captured once in a CUDA graph and replayed: every step of
    # this workload runs at the same context (seq_len is reset before each,
    # outside the timed region), so the replays repeat exactly the eager work
    # without the host round trips between its ~30 launches
    us_graph, graph_err = None, None
    try:
        seq.fill_(w.context)
        lens = [w.context] * w.batch
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):  # warm-up on the capture stream's side
            layer.step(xs[0], seq, lens)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        seq.fill_(w.context)
        lens = [w.context] * w.batch
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer.step(xs[0], seq, lens)
        torch.cuda.synchronize()
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        barrier(world)
        torch.cuda.synchronize()
        torch.cuda._sleep(int(5e7))
        for i in range(K):
            seq.fill_(w.context)
            flush.fill_(1)
            gev[i][0].record(stream)
            graph.replay()
            gev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        lk.device_status()
        us_graph = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in gev), world, device) / K * 1e3
        del graph
    except Exception as e:  # reported, not hidden: the eager number stands
        graph_err = f"{type(e).__name__}: {e}"[:200]
    us = us_graph if us_graph is not None else us_eager
    nbytes_w = sum(t.numel() * t.element_size() for t in (wts["W_Q"], wts["W_O"], wts["A"]))
    for name in ("gate", "up", "down"):
        d = wts[name]
        nbytes_w += sum(d[k].numel() * d[k].element_size() for k in ("W_D", "U", "V"))
    T = w.context + 1
    nbytes_c = w.batch * T * sum(r + r + 8 for r in rk)
    nbytes = nbytes_w + nbytes_c
    gbs = nbytes / (us * 1e-6) / 1e9
    hbm, peak_kind = peaks()
    if rank == 0:
        print(json.dumps({
            "mode": "layer", "metric": "W8A8 decoder-layer decode tokens/s", "value": w.batch * world / (us * 1e-6),
            "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup, "us_per_step": us,
            "higher_is_better": True, "scaling": "weak", "dtype": "int8/f32",
            "data": "synthetic (seeded W8A8 weights; random latent cache codes; shapes of the workload)",
            "config": {"workload": w.name, "batch": w.batch, "tokens": T,
                       "l2": "flushed before every step (256 MiB write, untimed)",
                       "launches": ("one CUDA graph per step (about 30 kernels), replayed" if us_graph is not None
                                    else "eager, one stream (about 30 kernel launches per step)")},
            "eager": {"us_per_step": us_eager, "value": w.batch * world / (us_eager * 1e-6)},
            "graph": ({"us_per_step": us_graph, "value": w.batch * world / (us_graph * 1e-6)}
                      if us_graph is not None else {"unavailable": graph_err}),
            "algorithmic_bytes_per_step": {"weights": nbytes_w, "latent_cache": nbytes_c},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_kind": peak_kind},
            "clocks": clocks.summary()}), flush=True)
    _finish(world)
    return 0


def run_rope(args):
    """The rotary-position decode (lk_latent_decode_attn_rope: keys rebuilt on
    chip, rotated) against the absorbed decode on the same caches, one layer
    of workloads 2-4, L2 flushed before every launch."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import rank_latent_kv_lk_b200 as lk
    from rank_latent_kv_lk_b200 import synth
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for e in ev:
            flush.fill_(1)
            e[0].record()
            fn()
            e[1].record()
        torch.cuda.synchronize()
        return statistics.median(e[0].elapsed_time(e[1]) * 1e3 for e in ev)

    hbm, peak_kind = peaks()
    lines = []
    for key in (2, 3, 4):
        w = WORKLOADS[key]
        rk, rv = synth.ranks(w)
        rk, rv = rk[0], rv[0]
        _, BK, BV = synth.factors(dataclasses.replace(w, act="bf16"), 0, rk, rv)
        BK, BV = BK.to(device), BV.to(device)
        T = w.context + 1
        g = torch.Generator(device=device)
        g.manual_seed(synth.seed_for(w, synth.CONTEXT))
        ck = lk.LatentCache(w.batch, rk, w.capacity, w.kind, w.group, device)
        cv = lk.LatentCache(w.batch, rv, w.capacity, w.kind, w.group, device, role="v")
        for c in (ck, cv):
            c.codes.copy_(torch.randint(0, 256, c.codes.shape, dtype=torch.uint8, device=device, generator=g))
            c.scales.copy_((torch.rand(c.scales.shape, device=device, generator=g) * 0.02 + 0.01).to(c.scales.dtype))
        q = torch.randn(w.batch, w.n_heads, w.head_dim, generator=g, device=device).to(torch.bfloat16)
        seq = torch.full((w.batch,), T, dtype=torch.int32, device=device)
        out = torch.empty(w.batch, w.n_heads, w.head_dim, dtype=torch.bfloat16, device=device)
        table = lk.rope_table(w.head_dim, w.capacity)
        absorbed_us = timed(lambda: lk.latent_decode_attn(ck, cv, q, BK, BV, seq, T, out=out), args.steps)
        rope_us = timed(lambda: lk.latent_decode_attn_rope(ck, cv, q, BK, BV, seq, T, table, out=out), args.steps)
        rb = lambda r: r if w.kind == "i8" else r // 2
        sb = lambda r: 4 if w.kind == "i8" else 2 * (-(-r // min(w.group, r)))
        cache_bytes = w.batch * T * (sum(rb(r) + sb(r) for r in rk) + sum(rb(r) + sb(r) for r in rv))
        flops = 2.0 * w.batch * T * sum(rk) * w.head_dim  # the key rebuild on the tensor cores
        lines.append({"workload": w.name, "batch": w.batch, "tokens": T, "absorbed_us": absorbed_us,
                      "rope_us": rope_us, "rope_cache_gbs": cache_bytes / rope_us / 1e3,
                      "rope_frac_of_measured_hbm": cache_bytes / rope_us / 1e3 / hbm,
                      "rope_key_rebuild_tflops": flops / rope_us / 1e6, "rope_over_absorbed": rope_us / absorbed_us})
        del ck, cv
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps({"mode": "rope", "l2": "flushed before every launch (256 MiB write, untimed)",
                          "peak_gbs": hbm, "peak_kind": peak_kind, "results": lines}))


def run_dense_compare(args):
    """The decode speed-up the pages report (latent attention vs flash decoding
    over dense K/V; the naive path that rebuilds K and V through memory), per
    workload, one layer, on this library's own kernels:
      latent : lk_latent_decode_attn over the latent cache;
      dense  : lk_dense_decode_attn over bf16 K and V of the same shapes;
      naive  : lk_latent_reconstruct_kv (K and V rebuilt into memory) followed
               by lk_dense_decode_attn;
    and, for context, torch's scaled_dot_product_attention (a library kernel)
    over the same dense K and V.  L2 flushed before every launch."""
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import rank_latent_kv_lk_b200 as lk
    from rank_latent_kv_lk_b200 import synth
    from rank_latent_kv_lk_b200.configs import WORKLOADS
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        torch.cuda._sleep(int(5e7))
        for e in ev:
            flush.fill_(1)
            e[0].record()
            fn()
            e[1].record()
        torch.cuda.synchronize()
        return statistics.median(e[0].elapsed_time(e[1]) * 1e3 for e in ev)

    hbm, peak_kind = peaks()
    lines = []
    for key in (2, 3, 4, 5):
        w = WORKLOADS[key]
        rk, rv = synth.ranks(w)
        rk, rv = rk[0], rv[0]
        _, BK, BV = synth.factors(dataclasses.replace(w, act="bf16"), 0, rk, rv)
        BK, BV = BK.to(device), BV.to(device)
        T = w.context + 1
        g = torch.Generator(device=device)
        g.manual_seed(synth.seed_for(w, synth.CONTEXT))
        ck = lk.LatentCache(w.batch, rk, w.capacity, w.kind, w.group, device)
        cv = lk.LatentCache(w.batch, rv, w.capacity, w.kind, w.group, device, role="v")
        for c in (ck, cv):
            c.codes.copy_(torch.randint(0, 256, c.codes.shape, dtype=torch.uint8, device=device, generator=g))
            c.scales.copy_((torch.rand(c.scales.shape, device=device, generator=g) * 0.02 + 0.01).to(c.scales.dtype))
        q = torch.randn(w.batch, w.n_heads, w.head_dim, generator=g, device=device).to(torch.bfloat16)
        seq = torch.full((w.batch,), T, dtype=torch.int32, device=device)
        out = torch.empty(w.batch, w.n_heads, w.head_dim, dtype=torch.bfloat16, device=device)
        latent_us = timed(lambda: lk.latent_decode_attn(ck, cv, q, BK, BV, seq, T, out=out), args.steps)
        Kd = torch.empty(w.batch, w.n_heads, w.capacity, w.head_dim, dtype=torch.bfloat16, device=device)
        Vd = torch.empty_like(Kd)
        naive_us = timed(lambda: (lk.reconstruct_kv(ck, cv, BK, BV, seq, T, w.head_dim, Kd, Vd),
                                  lk.dense_decode_attn(q, Kd, Vd, seq, T, out=out)), args.steps)
        recon_us = timed(lambda: lk.reconstruct_kv(ck, cv, BK, BV, seq, T, w.head_dim, Kd, Vd), args.steps)
        del ck, cv
        Kd.copy_(torch.randn(Kd.shape, generator=g, device=device).to(torch.bfloat16))
        Vd.copy_(torch.randn(Vd.shape, generator=g, device=device).to(torch.bfloat16))
        dense_us = timed(lambda: lk.dense_decode_attn(q, Kd, Vd, seq, T, out=out), args.steps)
        Ks, Vs = Kd[:, :, :T], Vd[:, :, :T]
        q4 = q.unsqueeze(2)
        sdpa_us = timed(lambda: torch.nn.functional.scaled_dot_product_attention(q4, Ks, Vs), args.steps)
        dense_bytes = 2 * w.batch * w.n_heads * T * w.head_dim * 2
        del Kd, Vd, Ks, Vs
        torch.cuda.empty_cache()
        lines.append({"workload": w.name, "layer": 0, "batch": w.batch, "tokens": T,
                      "latent_attn_us": latent_us, "dense_us": dense_us, "naive_us": naive_us,
                      "naive_reconstruct_us": recon_us, "library_sdpa_us": sdpa_us,
                      "dense_kv_bytes": dense_bytes, "dense_gbs": dense_bytes / (dense_us * 1e-6) / 1e9,
                      "dense_frac_of_measured_hbm": dense_bytes / (dense_us * 1e-6) / 1e9 / hbm,
                      "speedup_vs_dense": dense_us / latent_us, "speedup_vs_naive": naive_us / latent_us})
    if rank == 0:
        print(json.dumps({"mode": "dense-compare", "steps": args.steps,
                          "note": "latent, dense and naive on this library's kernels; torch SDPA for context",
                          "l2": "flushed before every launch (256 MiB write, untimed)",
                          "peak_gbs": hbm, "peak_kind": peak_kind, "results": lines}), flush=True)
    return 0


def _finish(world):
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.attn_only:
        return run_attn_only(args)
    if args.proj_only:
        return run_proj_only(args)
    if args.ffn_compare:
        return run_ffn_compare(args)
    if args.rope:
        return run_rope(args)
    if args.layer:
        return run_layer(args)
    if args.dense_compare:
        return run_dense_compare(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
