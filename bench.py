#!/usr/bin/env python
"""Benchmark: packed-KV decode attention (Block-GTQ / TQ-MSE) on B200.

One step = one decode step of a whole model's attention: for every layer, encode-append
the new token's key/value (TQ-MSE) into that layer's packed cache and run decode
attention of all query heads over the packed cache (split-K + log-sum-exp combine).
Each layer has its own cache, so a step reads every layer's cache once (far more than
the 126 MB L2). The step is captured in a CUDA graph and replayed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b|qwen3b|llama70b|tiny]
    python bench.py --impl reference ...      # the CPU oracle, timed on the host cores
    python bench.py --mode sweep              # decode over the 32q/8kv context x batch x rate grid
    python bench.py --mode encode             # tq_encode append throughput, 1 and 64 new tokens
    python bench.py --mode mae                # K-only logit error: block rates vs uniform rates

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
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

from packed_cache_decode_b200 import binding as B  # noqa: E402
from packed_cache_decode_b200 import sharding  # noqa: E402
from packed_cache_decode_b200 import synth  # noqa: E402

METRIC = "packed-KV decode attention: cached keys/s (HBM GB/s as % of B200 peak in roofline)"
UNIT = "keys/s"


PROFILE_KEYS = {"llama70b": "llama70b_b4_128k_k2v2", "llama8b": "llama8b_32k_k2v2", "qwen3b": "qwen3b_128k_k3v3"}


def _profiled_traffic(key: str):
    """DRAM bytes per launch of the split kernel from the committed ncu summary of this
    workload, or None when there is none or the kernel source has changed since."""
    import hashlib
    if key not in PROFILE_KEYS:
        return None
    prof = os.path.join(ROOT, "profiles", f"split_kernel_{PROFILE_KEYS[key]}.txt")
    src = os.path.join(ROOT, "packed_cache_decode_b200", "csrc", "decode_mma.cu")
    try:
        fields = dict(ln.split(":", 1) for ln in open(prof) if ln.startswith(("source_sha256_16:", "dram_bytes")))
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        if fields["source_sha256_16"].split()[0] != sha:
            return None
        return int(fields["dram_bytes_per_launch"].split()[0])
    except (OSError, KeyError, ValueError):
        return None


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples the GPU's SM clock and clock-event reasons through NVML every 10 ms on a
    host thread (reads only; nothing is set). mark() notes host times; summary(t0, t1)
    reports the samples taken between two marks."""

    REASONS = {"hw_slowdown": "HwSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
               "sw_thermal_slowdown": "SwThermalSlowdown", "sw_power_cap": "SwPowerCap",
               "hw_power_brake": "HwPowerBrakeSlowdown"}

    def __init__(self, device: torch.device):
        self.dev = device
        self.samples = []          # (host time, sm MHz, reason bits)
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nv = None
        self._h = None
        self.error = None

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            p = torch.cuda.get_device_properties(self.dev)
            try:
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                self._h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = nv.nvmlDeviceGetHandleByIndex(self.dev.index or 0)
            self._nv = nv
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
            t_end = time.monotonic() + 5.0
            while not self.samples and time.monotonic() < t_end:
                time.sleep(0.005)
        except Exception as e:       # no NVML: the line says so instead of guessing
            self.error = f"{type(e).__name__}: {e}"
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
                self.samples.append((time.monotonic(), mhz, bits))
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            self._stop.wait(0.01)

    @staticmethod
    def mark():
        return time.monotonic()

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        if self.error and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled: " + self.error], "samples": 0}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if not win:                    # timed region shorter than the sampling period
            later = [s for s in self.samples if s[0] >= t0]
            win = later[:1]
            window = "first sample after the timed region started"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for _, _, bits in win:
            for name, nvname in self.REASONS.items():
                mask = getattr(self._nv, "nvmlClocksEventReason" + nvname, 0)
                if bits & mask:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in win]), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win), "window": window}


# ------------------------------------------------------------------------ workload
class Model:
    """Per-layer packed caches and per-step inputs of one workload on one GPU. With a
    shard (sharding.Shard) the GPU holds only that shard's batch rows and KV heads (and
    the query heads that read them); rates are still allocated per layer over all heads."""

    def __init__(self, wl: synth.Workload, device: torch.device, seed_offset: int = 0, shard=None):
        self.wl = wl
        self.dev = device
        G = wl.h_q // wl.h_kv
        if shard is None:
            shard = sharding.Shard(0, wl.batch, 0, wl.h_kv)
        self.shard = shard
        self.heads = list(range(shard.h0, shard.h1))
        L = wl.length
        Bt, hkv = shard.b1 - shard.b0, shard.h1 - shard.h0
        hq = G * hkv
        self.batch, self.h_q, self.h_kv = Bt, hq, hkv
        self.capacity = 64 * math.ceil(L / 64)
        self.layers = []
        gen = torch.Generator(device=device)
        for layer in range(wl.layers):
            seed = wl.seed * 1000 + layer + seed_offset
            m = synth.make_layer_model(wl.h_q, wl.h_kv, seed)
            q_cal, k_cal = synth.make_calibration(m, 256, seed + 1, wl.theta)
            rates = B.plan_layer_rates(q_cal.numpy(), k_cal.numpy(), wl.k_bits)
            lay = B.Layout(rates, wl.v_bits, seed).upload(device.index)
            cache = torch.zeros(lay.cache_bytes(Bt, hkv, self.capacity), dtype=torch.uint8, device=device)
            gen.manual_seed(seed + 7919 * shard.b0 + 104729 * shard.h0)
            # prefill tokens 0..L-2 in bounded chunks (about 1 GB of fp32 draws at a time);
            # token L-1 is the one every step appends again
            chunk = int(max(64, min(16384, 1e9 // (Bt * hkv * 128 * 4 * 3))))
            lens0 = torch.zeros(Bt, dtype=torch.int32, device=device)
            for a in range(0, L, chunk):
                b = min(L, a + chunk)
                k, v = self._draw_kv(m, Bt, a, b, hkv, gen)
                n_enc = min(b, L - 1) - a
                if n_enc > 0:
                    lens0.fill_(a)
                    B.encode_append(lay, k[:, :n_enc].contiguous(), v[:, :n_enc].contiguous(), lens0, cache,
                                    self.capacity)
                if b == L:
                    k_new, v_new = k[:, -1:].contiguous(), v[:, -1:].contiguous()
                del k, v
            q = self._draw_q(m, Bt, hq, L - 1, gen)
            self.layers.append({
                "layout": lay, "cache": cache, "k_new": k_new, "v_new": v_new, "q": q,
                "out": torch.empty(Bt, hq, 128, dtype=torch.float32, device=device),
            })
        # all layers' step inputs (q, k_new, v_new) in one buffer and all outputs in another,
        # so that a host round trip of a step is one copy each way
        nq, nk = Bt * hq * 128, Bt * hkv * 128
        per = nq + 2 * nk
        self.inputs = torch.empty(wl.layers * per, dtype=wl.dtype, device=device)
        self.outputs = torch.empty(wl.layers, Bt, hq, 128, dtype=torch.float32, device=device)
        for i, x in enumerate(self.layers):
            base = i * per
            for key, off, n, shape in (("q", 0, nq, (Bt, hq, 128)), ("k_new", nq, nk, (Bt, 1, hkv, 128)),
                                       ("v_new", nq + nk, nk, (Bt, 1, hkv, 128))):
                view = self.inputs[base + off:base + off + n].view(shape)
                view.copy_(x[key])
                x[key] = view
            x["out"] = self.outputs[i]
        torch.cuda.synchronize(device)
        self.lens_before = torch.full((Bt,), L - 1, dtype=torch.int32, device=device)   # the step appends token L-1
        self.lens_after = torch.full((Bt,), L, dtype=torch.int32, device=device)
        ws = max(B.workspace_bytes(x["layout"], Bt, hq, hkv, L) for x in self.layers)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)
        self.bytes_per_step = sum(Bt * hkv * L * x["layout"].bytes_per_token for x in self.layers)
        self.keys_per_step = Bt * hkv * L * wl.layers

    def _draw_kv(self, m, Bt, a, b, hkv, gen):
        # Same recipe as synth.key_slice / value_slice (positions a..b-1), drawn on the device.
        dt = self.wl.dtype
        x = torch.randn(Bt, b - a, hkv, 128, generator=gen, device=self.dev)
        x *= torch.cat([m.k_scale, m.k_scale], 1)[self.heads].to(self.dev)[None, None]
        for i, h in enumerate(self.heads):
            x[:, :, i, m.outliers[h].to(self.dev)] *= m.outlier_gain
        x = _rope_dev(x, torch.arange(a, b, device=self.dev), self.wl.theta)
        v = torch.randn(Bt, b - a, hkv, 128, generator=gen, device=self.dev)
        return x.to(dt), v.to(dt)

    def _draw_q(self, m, Bt, hq, pos, gen):
        G = m.group
        qh = [h * G + j for h in self.heads for j in range(G)]
        x = torch.randn(Bt, 1, hq, 128, generator=gen, device=self.dev)
        x *= torch.cat([m.q_scale, m.q_scale], 1)[qh].to(self.dev)[None, None]
        for i, hh in enumerate(qh):
            x[:, :, i, m.outliers[hh // G].to(self.dev)] *= m.outlier_gain
        x = _rope_dev(x, torch.tensor([pos], device=self.dev), self.wl.theta)
        return x[:, 0].contiguous().to(self.wl.dtype)

    # kernel launches of one layer in a step: step-prep (encode + q-prep), the split kernel
    # and the log-sum-exp combine
    LAUNCHES_PER_LAYER = 3

    def step(self, stream):
        """Every layer: append the step's token and attend (one bgtq_decode_step call)."""
        for x in self.layers:
            B.decode_step(x["layout"], x["k_new"], x["v_new"], x["q"], x["cache"], self.lens_before, self.capacity,
                          self.wl.length, x["out"], self.workspace, stream=stream)

    def decode_layer(self, stream, i=0, reps=1):
        """The decode-attention call of layer i, reps times over the same cache."""
        x = self.layers[i]
        for _ in range(reps):
            B.decode_attention(x["layout"], x["q"], x["cache"], self.lens_after, self.capacity, self.wl.length,
                               x["out"], self.workspace, self.h_kv, stream=stream)

    def decode_only(self, stream):
        for x in self.layers:
            B.decode_attention(x["layout"], x["q"], x["cache"], self.lens_after, self.capacity, self.wl.length,
                               x["out"], self.workspace, self.h_kv, stream=stream)


def _rope_dev(x, pos, theta):
    inv = theta ** (-torch.arange(64, dtype=torch.float64, device=x.device) * 2.0 / 128)
    ang = pos.double()[:, None] * inv[None, :]
    c = torch.cos(ang)[None, :, None, :].float()
    s = torch.sin(ang)[None, :, None, :].float()
    a, b = x[..., :64], x[..., 64:]
    return torch.cat([a * c - b * s, b * c + a * s], dim=-1)


# ------------------------------------------------------------------------ oracle timing
def oracle_sample(wl: synth.Workload, budget_s: float, max_tokens: int = 16384):
    """Time the CPU oracle on whole (batch row, KV head) units of one layer of the
    workload: encode the new token, then unpack + reconstruct + attend over the cache.
    The sample is bounded: each unit's context is the workload's first max_tokens tokens
    (the oracle's cost per cached key does not depend on the context length)."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    m = synth.make_layer_model(wl.h_q, wl.h_kv, wl.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, wl.seed + 1, wl.theta)
    rates = O.greedy_rates(O.block_energy(q_cal.double().numpy(), k_cal.double().numpy()),
                           O.lloyd_max_mse_table(), 1, 4, 64 * wl.k_bits)
    lay = O.make_layout(rates, wl.v_bits, wl.seed)
    G = wl.h_q // wl.h_kv
    L = min(wl.length, max_tokens)
    cap = 64 * math.ceil(L / 64)
    prepared = []
    for h in range(min(2, wl.h_kv)):
        k = synth.key_slice(m, 0, h, L, 0, wl.seed, wl.theta).double().numpy()
        v = synth.value_slice(m, 0, h, L, wl.seed).double().numpy()
        q = torch.stack([synth.query_slice(m, 0, h * G + i, 1, L - 1, wl.seed, wl.theta)[0]
                         for i in range(G)]).double().numpy()
        prepared.append((k, v, q, O.pack(lay, O.encode(lay, k[:-1], v[:-1]), cap)))
    units, keys, elapsed = 0, 0, 0.0
    while elapsed < budget_s:
        k, v, q, buf = prepared[units % len(prepared)]
        t0 = time.perf_counter()
        new = O.encode(lay, k[-1:], v[-1:])                        # the step's append
        u = O.unpack(lay, buf, L - 1)
        for key in ("k_codes", "v_codes"):
            u[key] = np.concatenate([u[key], new[key]])
        u["k_norms"] = np.concatenate([u["k_norms"], new["k_norms"].astype(np.float32)])
        u["v_norm"] = np.concatenate([u["v_norm"], new["v_norm"].astype(np.float32)])
        kh, vh = O.reconstruct(lay, u["k_codes"], u["k_norms"], u["v_codes"], u["v_norm"])
        O.attention(q, kh, vh, 1 / math.sqrt(128))
        elapsed += time.perf_counter() - t0
        units += 1
        keys += L
    return {"value": keys / elapsed, "unit": UNIT, "cores": cores, "kind": "oracle",
            "threads": f"numpy with {cores} BLAS thread(s) for the matrix products; the oracle's Python loops run "
                       f"on one core",
            "sample": f"{units} (batch row, KV head) unit passes over {len(prepared)} distinct unit(s) of one "
                      f"layer, the first {L} cached tokens of the workload each: append 1 token + decode "
                      f"attention, {elapsed:.1f} s"}


# ------------------------------------------------------------------------ sweep / encode modes
def _time_graph(fn, stream, reps):
    with torch.cuda.stream(stream):
        for _ in range(2):
            fn(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del g
    return ms


def run_sweep(args):
    """Decode attention over the 32q/8kv grid; each point cycles enough per-layer caches
    to exceed L2 (>= 256 MB per replay, at most 32 layers)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = _peaks()
    stream = torch.cuda.Stream()
    for wl in synth.sweep_workloads():
        bpt = 128 * wl.k_bits // 8 + 128 * wl.v_bits // 8 + 20
        per_layer = wl.batch * wl.h_kv * wl.length * bpt
        layers = int(min(32, max(1, math.ceil(256e6 / per_layer))))
        if per_layer * layers > 40e9:
            continue
        w = synth.Workload(**{**wl.__dict__, "layers": layers})
        model = Model(w, dev)
        ms = _time_graph(model.decode_only, stream, max(5, args.steps))
        keys = w.batch * w.h_kv * w.length * layers
        gbs = model.bytes_per_step / (ms * 1e-3) / 1e9
        print(json.dumps({"mode": "sweep", "workload": w.name, "layers_cycled": layers,
                          "us_per_layer": ms * 1e3 / layers, "keys_per_s": keys / (ms * 1e-3), "GBs": gbs,
                          "hbm_frac": gbs / peak, "peak_kind": peak_kind}), flush=True)
        del model
        torch.cuda.empty_cache()


def run_encode(args):
    """tq_encode append throughput on the 32q/8kv shape (K2V2 layout), n_new in {1, 64}."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream()
    m = synth.make_layer_model(32, 8, 4)
    q_cal, k_cal = synth.make_calibration(m, 256, 5, 5e5)
    rates = B.plan_layer_rates(q_cal.numpy(), k_cal.numpy(), 2)
    lay = B.Layout(rates, 2, 4).upload(0)
    for batch in (1, 8, 32):
        for n_new in (1, 64):
            cap = 4096
            cache = torch.zeros(lay.cache_bytes(batch, 8, cap), dtype=torch.uint8, device=dev)
            k = torch.randn(batch, n_new, 8, 128, device=dev).to(torch.bfloat16)
            v = torch.randn_like(k)
            lens = torch.full((batch,), 1000, dtype=torch.int32, device=dev)
            ms = _time_graph(lambda st: B.encode_append(lay, k, v, lens, cache, cap, stream=st), stream,
                             max(20, args.steps))
            toks = batch * n_new
            print(json.dumps({"mode": "encode", "batch": batch, "n_new": n_new, "h_kv": 8, "rates": "K2V2",
                              "us_per_call": ms * 1e3, "tokens_per_s": toks / (ms * 1e-3),
                              "token_heads_per_s": toks * 8 / (ms * 1e-3)}), flush=True)


def run_mae(args):
    """K-only logit error of the block rate allocation against uniform rates at the same
    bit budget, on the 8B- and 3B-shaped generators (8192 cached tokens, one layer): the
    logits come from bgtq_decode_scores over each packed cache, the exact ones from the
    unquantised keys (fp64). Reports the mean absolute logit error of both layouts, and of
    the block allocation with norm correction and/or fp16 norms and of the allocation that
    may leave blocks uncoded (rates from 0) and of an allocation per KV head (each head its
    own layout, all heads in one call through a layout set), with each layout's
    resident bytes per (token, KV head) and its footprint ratio to an fp16 K+V record
    (512 bytes)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    for name in ("llama8b", "qwen3b"):
        base = synth.WORKLOADS[name]
        wl = synth.Workload(**{**base.__dict__, "length": 8192, "batch": 1, "layers": 1})
        m = synth.make_layer_model(wl.h_q, wl.h_kv, wl.seed)
        q_cal, k_cal = synth.make_calibration(m, 256, wl.seed + 1, wl.theta)
        rates = B.plan_layer_rates(q_cal.numpy(), k_cal.numpy(), wl.k_bits)
        q, k, v = synth.make_cache_inputs(m, 1, wl.length, wl.seed, wl.theta, torch.float32)
        scale = 1.0 / math.sqrt(128)
        G = wl.h_q // wl.h_kv
        exact = torch.einsum("hgd,htd->hgt", q[0].view(wl.h_kv, G, 128).double(), k[0].transpose(0, 1).double())
        exact = (exact * scale).reshape(wl.h_q, wl.length).to(dev)
        line = {"mode": "mae", "workload": wl.name, "tokens": wl.length, "k_bits": wl.k_bits,
                "block_rates": {str(r): int((rates == r).sum()) for r in sorted(set(rates.tolist()))}}
        uni = np.full(64, wl.k_bits)
        rates0 = B.plan_layer_rates(q_cal.numpy(), k_cal.numpy(), wl.k_bits, min_rate=0)
        line["block_rates_from_0"] = {str(r): int((rates0 == r).sum()) for r in sorted(set(rates0.tolist()))}
        variants = (("block_gtq", rates, False, False), ("uniform", uni, False, False),
                    ("block_gtq_rate0", rates0, False, False),
                    ("block_gtq_nc", rates, True, False), ("block_gtq_fp16", rates, False, True),
                    ("block_gtq_nc_fp16", rates, True, True), ("uniform_nc", uni, True, False))
        for tag, rr, nc, fp16 in variants:
            lay = B.Layout(rr, wl.v_bits, wl.seed, nc, fp16).upload(0)
            cap = wl.length
            cache = torch.zeros(lay.cache_bytes(1, wl.h_kv, cap), dtype=torch.uint8, device=dev)
            lens = torch.zeros(1, dtype=torch.int32, device=dev)
            B.encode_append(lay, k.to(dev), v.to(dev), lens, cache, cap)
            lens.fill_(wl.length)
            ws = torch.empty(B.workspace_bytes(lay, 1, wl.h_q, wl.h_kv, wl.length), dtype=torch.uint8, device=dev)
            sc = torch.empty(1, wl.h_q, wl.length, dtype=torch.float32, device=dev)
            B.decode_scores(lay, q.to(dev), cache, lens, cap, wl.length, sc, ws, wl.h_kv)
            torch.cuda.synchronize()
            line[f"mae_{tag}"] = float((sc[0].double() - exact).abs().mean())
            line[f"bytes_per_token_{tag}"] = lay.bytes_per_token
            line[f"footprint_x_{tag}"] = round(2 * 128 * 2 / lay.bytes_per_token, 3)
            assert lay.status() == 0
        # an allocation per KV head: every head's own rates and layout, all heads in one
        # encode and one scores call through a layout set
        per_head = B.plan_head_rates(q_cal.numpy(), k_cal.numpy(), wl.k_bits)
        heads = [B.Layout(per_head[h], wl.v_bits, wl.seed).upload(0) for h in range(wl.h_kv)]
        S = B.LayoutSet(heads)
        cache = torch.zeros(S.cache_bytes(1, wl.length), dtype=torch.uint8, device=dev)
        lens = torch.zeros(1, dtype=torch.int32, device=dev)
        B.encode_append_heads(S, k.to(dev), v.to(dev), lens, cache, wl.length)
        lens.fill_(wl.length)
        ws = torch.empty(B.workspace_bytes(heads[0], 1, wl.h_q, wl.h_kv, wl.length), dtype=torch.uint8, device=dev)
        sc = torch.empty(1, wl.h_q, wl.length, dtype=torch.float32, device=dev)
        B.decode_scores_heads(S, q.to(dev), cache, lens, wl.length, wl.length, sc, ws)
        torch.cuda.synchronize()
        assert S.status() == 0
        err = float((sc[0].double() - exact).abs().sum())
        nbytes = sum(lay.bytes_per_token for lay in heads)
        line["mae_block_gtq_per_head"] = err / (wl.h_q * wl.length)
        line["bytes_per_token_block_gtq_per_head"] = nbytes / wl.h_kv
        line["reduction"] = 1.0 - line["mae_block_gtq"] / line["mae_uniform"]
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama70b", choices=list(synth.WORKLOADS))
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-others", action="store_true", help="skip the 8B- and 3B-shaped lines of the default run")
    ap.add_argument("--shard", action="store_true",
                    help="N > 1: split one workload's (batch row, KV head) units over the ranks (strong scaling) "
                         "instead of running independent replicas")
    ap.add_argument("--mode", default="step", choices=["step", "sweep", "encode", "mae"])
    args = ap.parse_args()
    if args.mode == "sweep":
        return run_sweep(args)
    if args.mode == "encode":
        return run_encode(args)
    if args.mode == "mae":
        return run_mae(args)
    wl = synth.WORKLOADS[args.workload]
    if args.layers:
        wl = synth.Workload(**{**wl.__dict__, "layers": args.layers})

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        per_step = []
        for _ in range(args.warmup):
            oracle_sample(wl, args.cpu_budget / max(1, args.steps + args.warmup))
        for _ in range(args.steps):
            per_step.append(oracle_sample(wl, args.cpu_budget / max(1, args.steps)))
        v = statistics.median([p["value"] for p in per_step])
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": wl.name, "layers": wl.layers},
                "cpu_baseline": {"value": v, "unit": UNIT, "cores": per_step[0]["cores"], "kind": "oracle",
                                 "sample": "per step: " + per_step[0]["sample"]},
                "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    shard = sharding.shard_units(wl.batch, wl.h_kv, rank, world) if args.shard else None
    model = Model(wl, dev, seed_offset=0 if args.shard else rank * 100000, shard=shard)
    stream = torch.cuda.Stream(device=dev)

    def barrier():
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)

    clk = ClockSampler(dev).start()
    r = measure(model, stream, args.steps, args.warmup, barrier, clk)
    clk.stop()
    clocks = clk.summary(r["t_on"], r["t_off"])

    times = torch.tensor([r["step_ms"], r["dec_ms"], r["e2e_ms"], r["l2_ms"]], dtype=torch.float64, device=dev)
    totals = torch.tensor([float(model.keys_per_step), float(model.bytes_per_step)], dtype=torch.float64, device=dev)
    if pg:
        pg.all_reduce(times, op=pg.ReduceOp.MAX)
        pg.all_reduce(totals, op=pg.ReduceOp.SUM)
    step_ms, dec_ms, e2e_ms, l2_ms = times.tolist()
    keys, total_bytes = totals.tolist()

    if rank == 0:
        peak, peak_kind = _peaks()
        dec_bytes = model.bytes_per_step / wl.layers
        achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
        layer_mb = dec_bytes / 1e6
        line = {
            "metric": METRIC, "value": keys / (step_ms * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "strong" if args.shard else "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "layers": wl.layers, "batch": wl.batch, "context": wl.length,
                       "h_q": wl.h_q, "h_kv": wl.h_kv, "rates": f"K{wl.k_bits}V{wl.v_bits}",
                       "bytes_per_token_head": model.layers[0]["layout"].bytes_per_token,
                       "step": "per layer: bgtq_decode_step (append 1 token + decode attention); CUDA graph",
                       "l2": f"inputs larger than L2: {model.bytes_per_step / 1e6:.0f} MB of packed caches per step "
                             f"on each GPU (one cache per layer)",
                       "parallelism": (f"(batch row, KV head) units sharded over {world} GPU(s), no collective on the "
                                       f"data path" if args.shard else
                                       f"replicas x{world} (independent sequences per GPU)")},
            "gbs": total_bytes / (step_ms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": _profiled_traffic(args.workload),
                         "kernel": "decode attention call per layer (q-prep -> split -> combine, PDL-chained)",
                         "bytes_per_launch": dec_bytes, "peak_kind": peak_kind},
            "l2_warm": {"us_per_call": l2_ms * 1e3, "GBs": dec_bytes / (l2_ms * 1e-3) / 1e9,
                        "note": f"layer 0's decode call repeated over the same {layer_mb:.0f} MB cache"
                                + (" (fits the 126 MB L2)" if layer_mb < 126 else " (larger than L2: read from HBM)")},
            "clocks": clocks,
            "gpu_launches": args.steps * wl.layers * Model.LAUNCHES_PER_LAYER,
            "e2e": {"value": keys / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": r["h2d"],
                    "d2h_bytes_per_step": r["d2h"]},
        }
        if world == 1 and not args.no_others and args.workload == "llama70b":
            line["other_workloads"] = other_workloads(args, dev, stream, barrier, peak)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_sample(wl, args.cpu_budget)
            line["codes_vs_oracle"] = codes_vs_oracle(wl, dev)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def measure(model, stream, steps, warmup, barrier, clk=None):
    """Device times (CUDA events on the launching stream) of one model: the decode step
    (all layers, CUDA graph), the decode-attention calls alone (graph over all layers),
    layer 0's call repeated over one cache (L2-warm when it fits), and the same step end to
    end with host buffers (one pinned copy each way per step inside the timed region)."""
    dev = model.dev
    with torch.cuda.stream(stream):
        for _ in range(2):
            model.step(stream)
    torch.cuda.synchronize(dev)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        model.step(stream)
    g_dec = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_dec, stream=stream):
        model.decode_only(stream)
    reps = 20
    g_l2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_l2, stream=stream):
        model.decode_layer(stream, 0, reps)
    torch.cuda.synchronize(dev)

    def timed(graph, n, pre=3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(pre):
                graph.replay()
            e0.record(stream)
            for _ in range(n):
                graph.replay()
            e1.record(stream)
        barrier()
        return e0.elapsed_time(e1) / n

    with torch.cuda.stream(stream):
        for _ in range(max(3, warmup)):
            g_step.replay()
    barrier()
    t_on = clk.mark() if clk else 0.0
    step_ms = timed(g_step, steps, pre=0)
    t_off = clk.mark() if clk else 0.0
    dec_ms = timed(g_dec, steps) / model.wl.layers
    l2_ms = timed(g_l2, max(3, steps // 2)) / reps

    # end to end through the public API with host buffers (pinned), copies inside the timing:
    # every step copies all layers' inputs in and all outputs back, one copy each way
    h_in = model.inputs.cpu().pin_memory()
    h_out = torch.empty_like(model.outputs, device="cpu").pin_memory()

    def e2e_step():
        model.inputs.copy_(h_in, non_blocking=True)
        g_step.replay()
        h_out.copy_(model.outputs, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / steps
    del g_step, g_dec, g_l2
    return {"step_ms": step_ms, "dec_ms": dec_ms, "l2_ms": l2_ms, "e2e_ms": e2e_ms, "t_on": t_on, "t_off": t_off,
            "h2d": h_in.numel() * h_in.element_size(), "d2h": h_out.numel() * h_out.element_size()}


def other_workloads(args, dev, stream, barrier, peak):
    """The 8B- and 3B-shaped layers measured the same way in the same run (their whole
    steps, the decode call's HBM fraction, the L2-warm single-layer call)."""
    out = {}
    for key in ("llama8b", "qwen3b"):
        wl = synth.WORKLOADS[key]
        model = Model(wl, dev)
        r = measure(model, stream, max(5, args.steps), args.warmup, barrier)
        dec_bytes = model.bytes_per_step / wl.layers
        out[key] = {"workload": wl.name, "layers": wl.layers, "ms_per_step": r["step_ms"],
                    "keys_per_s": model.keys_per_step / (r["step_ms"] * 1e-3),
                    "decode_call_us": r["dec_ms"] * 1e3, "decode_call_GBs": dec_bytes / (r["dec_ms"] * 1e-3) / 1e9,
                    "frac": dec_bytes / (r["dec_ms"] * 1e-3) / 1e9 / peak,
                    "l2_warm_us_per_call": r["l2_ms"] * 1e3,
                    "l2_warm_GBs": dec_bytes / (r["l2_ms"] * 1e-3) / 1e9,
                    "e2e_keys_per_s": model.keys_per_step / (r["e2e_ms"] * 1e-3),
                    "bytes_per_token_head": model.layers[0]["layout"].bytes_per_token}
        del model
        torch.cuda.empty_cache()
    return out


def codes_vs_oracle(wl, dev, units=2, tokens=4096):
    """Near-threshold code statistics on a bounded sample: the GPU encodes (batch row 0,
    KV heads 0..units-1) x tokens of the workload's generator; the oracle encodes the same
    inputs. Codes may differ only where the oracle's rotated value lies within 1e-6 of a
    decision threshold; reports how many such coordinates there are and how many differ."""
    import oracle as O
    m = synth.make_layer_model(wl.h_q, wl.h_kv, wl.seed)
    q_cal, k_cal = synth.make_calibration(m, 256, wl.seed + 1, wl.theta)
    rates = O.greedy_rates(O.block_energy(q_cal.double().numpy(), k_cal.double().numpy()),
                           O.lloyd_max_mse_table(), 1, 4, 64 * wl.k_bits)
    olay = O.make_layout(rates, wl.v_bits, wl.seed)
    lay = B.Layout(rates, wl.v_bits, wl.seed).upload(dev.index)
    n = min(tokens, wl.length)
    k = torch.stack([synth.key_slice(m, 0, h, n, 0, wl.seed, wl.theta) for h in range(units)], 1).to(wl.dtype)
    v = torch.stack([synth.value_slice(m, 0, h, n, wl.seed) for h in range(units)], 1).to(wl.dtype)
    cap = 64 * math.ceil(n / 64)
    cache = torch.zeros(lay.cache_bytes(1, units, cap), dtype=torch.uint8, device=dev)
    lens = torch.zeros(1, dtype=torch.int32, device=dev)
    B.encode_append(lay, k[None].to(dev), v[None].to(dev), lens, cache, cap)
    got_all = cache.cpu().numpy()
    per = cap // 64 * olay.tile_bytes
    coords = near = near_diff = elsewhere = 0
    for h in range(units):
        enc = O.encode(olay, k[:, h].double().numpy(), v[:, h].double().numpy())
        want = O.unpack(olay, O.pack(olay, enc, cap), n)
        got = O.unpack(olay, got_all[h * per:(h + 1) * per], n)
        mk, mv = enc["k_margin"] < 1e-6, enc["v_margin"] < 1e-6
        dk, dv = got["k_codes"] != want["k_codes"], got["v_codes"] != want["v_codes"]
        coords += mk.size + mv.size
        near += int(mk.sum() + mv.sum())
        near_diff += int((dk & mk).sum() + (dv & mv).sum())
        elsewhere += int((dk & ~mk).sum() + (dv & ~mv).sum())
    return {"coords": coords, "near_threshold": near, "near_threshold_coded_differently": near_diff,
            "differ_elsewhere": elsewhere, "sample": f"batch row 0, KV heads 0..{units - 1}, {n} tokens, one layer"}


if __name__ == "__main__":
    main()
