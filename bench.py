#!/usr/bin/env python
"""Benchmark of the hybrid-head KV attention path on B200.

Headline workload (N = 1): decode attention of a Llama-3-8B-shaped GQA model (32
layers; per layer 32 q / 8 kv heads, d 128, 4 retrieval + 4 streaming kv heads, S 16,
W 512, bf16) at a 128K-token context, batch 1.  One step = one new token through the
32 layer caches (32 x 0.27 GB of K/V, far larger than L2, so no L2 flush is needed):
per layer, append the token's K/V and run decode attention -- the whole decode path
(append/evict, retrieval split-KV, streaming sink+ring, merge), through
duo_append_decode (one fused launch per layer at batch 1).  value = algorithmic HBM
bytes of the decode attention per step / step time (GB/s), the step timed with no
events between its launches.  The K steps the driver asks for are timed as one region;
the region is repeated (at least 5 times, and until about half a second of GPU time
is covered) and value is the median region, with the spread reported beside it.

"workloads" holds every decode configuration on the same footing (Llama-2-7B MHA 32K
at batch 1 and 8, Llama-3-8B GQA 128K at batch 1 and 4, the 1M-token 32-layer stack
with INT4 retrieval heads, Llama-3 128K with FP8 retrieval heads, a ragged batch of 8
Llama-3 sequences from 2K to 128K tokens in the paged pool, and Llama-2 32K with the
pool's 32-layers-per-launch step): 5 regions of at least 100 ms of GPU time each,
median and spread, its roofline against the measured HBM peak, the clocks seen, and
the fp64 oracle timed on the host cores on a bounded sample of the same workload.  The chunked
pre-fill (256K prompt in 32K chunks, same shape; at least 5 runs) is reported under
"prefill" with an oracle baseline extrapolated from sampled query rows, and the
identification-phase gated forward (32K tokens) under "gated".

roofline.traffic is the DRAM traffic per launch from a committed ncu capture, reported
while the sources of the kernels the workload runs still hash to the recorded value.

--impl reference times the fp64 CPU oracle on the host cores, K steps after W warm-up
steps, each step a bounded sample of the headline step (the oracle's decode of a few
of its layers).  Under torchrun every rank runs an independent replica (the path does
not shard); value sums the ranks' bytes over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn achieved HBM GB/s + μs/token/layer at 128K; prefill TFLOP/s"
WORKLOAD = "llama3-8b-gqa-decode-128k-b1"
HQ, HKV, D, NRET, S, W = 32, 8, 128, 4, 16, 512
CTX = 131072
PREFILL_LEN, PREFILL_CHUNK = 262144, 32768
LAYERS = 32  # Llama-2-7B and Llama-3-8B both have 32 layers

# decode workloads: (q heads, kv heads, retrieval kv heads, context, batch, layers, retrieval format);
# a step visits the `layers` caches in turn (one new token through the model)
DECODE_WORKLOADS = {
    "llama3-8b-gqa-decode-128k-b1": (32, 8, 4, 131072, 1, LAYERS, "same"),
    "llama3-8b-gqa-decode-128k-b4": (32, 8, 4, 131072, 4, LAYERS, "same"),
    "llama2-7b-mha-decode-32k-b1": (32, 32, 8, 32768, 1, LAYERS, "same"),
    "llama2-7b-mha-decode-32k-b8": (32, 32, 8, 32768, 8, LAYERS, "same"),
    "llama3-8b-gqa-decode-1m-int4-32l": (32, 8, 4, 1 << 20, 1, LAYERS, "int4"),
    "llama3-8b-gqa-decode-128k-fp8-b1": (32, 8, 4, 131072, 1, LAYERS, "fp8"),
}
# pool (ragged batch) workloads: (q heads, kv heads, retrieval kv heads, contexts of the
# sequences, layers, layers per decode_step call); every step appends one token to every
# sequence on every layer and attends
POOL_WORKLOADS = {
    "llama3-8b-gqa-decode-ragged-8seq-32l": (32, 8, 4, [2048, 4096, 8192, 16384, 32768, 65536, 98304, 131072],
                                             LAYERS, 1),
    "llama2-7b-mha-decode-32k-b1-pool-32l-per-launch": (32, 32, 8, [32768], LAYERS, LAYERS),
}
REGIONS = 5              # timed regions per workload (median and spread reported)
REGION_MS = 100.0        # GPU time per region of a workload entry, at least
HEADLINE_TOTAL_MS = 500.0  # headline: regions of K steps until about this much is timed
MAX_HEADLINE_REGIONS = 25
MAX_REGION_STEPS = 400


def decode_bytes(len_, B=1, Hr=NRET, Hs=HKV - NRET, Hq=HQ, d=D, fmt="same", S=S, W=W):
    """Algorithmic HBM bytes of one decode-attention call: every visible K and V row
    once (bf16 rows, INT4 codes plus fp16 scale/zero, or FP8 codes plus an fp32 scale),
    the queries, the outputs and the lse."""
    kv = 2 * d * 2
    rkv = {"int4": 2 * (d // 2 + 4), "fp8": 2 * (d + 4)}.get(fmt, kv)
    return B * (Hr * len_ * rkv + Hs * min(len_, S + W) * kv) + B * Hq * d * 2 * 2 + B * Hq * 4


def visible_pairs(i, retrieval, S=S, W=W):
    """Keys visible to the query at absolute position i (causal, or sinks + window)."""
    if retrieval:
        return i + 1
    return min(i + 1, S) + min(W, max(0, i + 1 - S))


def prefill_flops(L=PREFILL_LEN, Hq=HQ, d=D, G=HQ // HKV, nret=NRET):
    """Algorithmic FLOPs of the full pre-fill: 4 d per visible (query, key) pair."""
    retr_pairs = L * (L + 1) // 2
    sw = S + W
    # streaming rows: i+1 keys while i < S+W, then S+W
    strm_pairs = sw * (sw + 1) // 2 + (L - sw) * sw if L > sw else L * (L + 1) // 2
    return 4 * d * G * (nret * retr_pairs + (HKV - nret) * strm_pairs)


def gated_flops(L, Hq=HQ, d=D):
    """Algorithmic FLOPs of the gated forward over one sequence: every query head pays
    4 d per causally visible pair (full term) plus 4 d per Lambda-visible pair."""
    causal = L * (L + 1) // 2
    sw = S + W
    lam = sw * (sw + 1) // 2 + (L - sw) * sw if L > sw else causal
    return 4 * d * Hq * (causal + lam)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def spread(values):
    """Median, min, max and (max - min) / median in percent of a list of region values."""
    med = statistics.median(values)
    return {"median": round(med, 3), "min": round(min(values), 3), "max": round(max(values), 3),
            "spread_pct": round(100.0 * (max(values) - min(values)) / med, 2) if med else None, "n": len(values)}


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    def __init__(self, index=0):
        self.index, self.proc, self.lines = index, None, []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _hash_files(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "head_split_kv_duo_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def kernel_hash(workload):
    """Hash of the sources of the decode kernels a workload runs: recorded DRAM traffic
    is void once they change."""
    files = ["k_decode_tc.cu", "tcgen05.cuh", "decode_merge.cuh", "device_common.cuh", "duo_internal.h"]
    if "int4" in workload:
        files.append("k_decode_int4_tc.cu")
    if "fp8" in workload:
        files.append("k_decode_fp8_tc.cu")
    return _hash_files(files)


def prefill_kernel_hash():
    return _hash_files(["k_prefill_tc.cu", "tcgen05.cuh", "device_common.cuh", "duo_internal.h"])


def _record(name):
    path = os.path.join(ROOT, "profiles", name)
    return json.load(open(path)) if os.path.exists(path) else {}


def recorded_traffic(workload):
    """DRAM bytes (read + write) per decode launch from the committed ncu summary of
    this workload, when it was taken on the current kernel source."""
    rec = _record("decode_traffic.json").get(workload)
    if not rec or rec.get("kernel_hash") != kernel_hash(workload):
        return None
    return rec.get("dram_bytes_per_launch")


def recorded_prefill_counters():
    """ncu counters of one pre-fill launch (tensor pipe, DRAM) recorded on the current
    kernel source, or None."""
    rec = _record("prefill_counters.json")
    if not rec or rec.get("kernel_hash") != prefill_kernel_hash():
        return None
    return rec


# ---------------------------------------------------------------- our arm

def reduce_over_ranks(dist, ms, nbytes, device):
    """Whole-job timing over the ranks: the slowest rank's time and the bytes of all
    ranks (every rank takes both collectives, in the same order)."""
    if not dist:
        return ms, float(nbytes)
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    b = torch.tensor([float(nbytes)], device=device, dtype=torch.float64)
    dist.all_reduce(b)
    return float(t.item()), float(b.item())


def launches_per_layer(B, fmt, Hs):
    """Kernel launches of one duo_append_decode call (see include/duo.h)."""
    if fmt == "same":
        return (1, "fused append+decode") if B == 1 else (2, "append, then decode")
    return (3 if Hs > 0 else 2), f"append, bf16 streaming-head decode, {fmt.upper()} retrieval-head decode"


class DecodeRun:
    """One decode workload: a cache of `layers` layers filled to `ctx` tokens and the
    per-step inputs; step(i) appends token i to every layer and attends."""

    def __init__(self, name, dev, extra_tokens, nstep_in, layers=0):
        import torch

        from head_split_kv_duo_b200 import inputs
        from head_split_kv_duo_b200.duo import DuoCache

        self.name = name
        self.Hq, self.Hkv, self.nret, self.ctx, self.B, self.layers, self.fmt = DECODE_WORKLOADS[name]
        if layers:
            self.layers = layers
        self.Hr, self.Hs = self.nret, self.Hkv - self.nret
        self.dev = dev
        max_len = self.ctx + extra_tokens
        mask = inputs.retrieval_mask(self.layers, self.Hkv, self.nret, seed=1)
        self.cache = DuoCache(self.layers, self.Hkv, D, mask, S, W, max_len, batch=self.B, q_heads=self.Hq,
                              dtype=torch.bfloat16, retr_fmt=self.fmt, device=dev)
        # fill each layer to ctx tokens (seeded N(0,1) K/V), in pieces of at most 2^18 tokens
        piece = min(self.ctx, 1 << 18)
        for layer in range(self.layers):
            for t0 in range(0, self.ctx, piece):
                n = min(piece, self.ctx - t0)
                k = inputs.randn((self.B, n, self.Hkv, D), 100 + 1000 * layer + 2 * t0 // piece, device=dev)
                v = inputs.randn((self.B, n, self.Hkv, D), 101 + 1000 * layer + 2 * t0 // piece, device=dev)
                self.cache.append_kv(layer, k, v)
                del k, v
        torch.cuda.synchronize()
        # per-step inputs (q, k, v of the new token for every layer), reused cyclically
        self.nin = nstep_in
        self.qs = inputs.randn((nstep_in, self.layers, self.B, self.Hq, D), 7, device=dev)
        self.ks = inputs.randn((nstep_in, self.layers, self.B, 1, self.Hkv, D), 8, device=dev)
        self.vs = inputs.randn((nstep_in, self.layers, self.B, 1, self.Hkv, D), 9, device=dev)
        self.out = torch.empty(self.layers, self.B, self.Hq, D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(self.layers, self.B, self.Hq, dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream()
        self.lpl, self.launch_desc = launches_per_layer(self.B, self.fmt, self.Hs)

    def nbytes_of(self, n):
        return decode_bytes(n, B=self.B, Hr=self.Hr, Hs=self.Hs, Hq=self.Hq, fmt=self.fmt)

    def step(self, i, ev=None):
        import torch
        j = i % self.nin
        nbytes = 0
        for layer in range(self.layers):
            n = self.cache.len(layer) + 1
            if ev is not None:
                ev[0].record(self.stream)
            self.cache.append_decode(layer, self.qs[j, layer], self.ks[j, layer], self.vs[j, layer],
                                     out=self.out[layer], lse=self.lse[layer], stream=self.stream)
            if ev is not None:
                ev[1].record(self.stream)
                ev[2].append((ev[0], ev[1]))
                ev[0] = torch.cuda.Event(enable_timing=True)
                ev[1] = torch.cuda.Event(enable_timing=True)
            nbytes += self.nbytes_of(n)
        return nbytes

    def region(self, first, steps, dist=None):
        """Times `steps` steps as one region (synchronize and barrier on both sides);
        returns (ms, bytes)."""
        import torch
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        t0.record(self.stream)
        nbytes = 0
        for i in range(first, first + steps):
            nbytes += self.step(i)
        t1.record(self.stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        return t0.elapsed_time(t1), nbytes

    def close(self):
        import torch
        assert self.cache.device_status() == 0, "device status word set"
        self.cache.close()
        del self.cache, self.qs, self.ks, self.vs
        torch.cuda.empty_cache()


def roofline_entry(name, per_launch_bytes, call_ms, hbm_peak, peak_src, launch_desc):
    achieved = per_launch_bytes / (call_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "decode", "achieved": round(achieved, 1), "peak": hbm_peak,
            "peak_source": f"{peak_src} hbm_gbs (burst copy)", "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
            "frac_of_8tbs_spec": round(achieved / 8000.0, 4), "traffic": recorded_traffic(name),
            "algorithmic_bytes_per_launch": int(per_launch_bytes), "avg_launch_us": round(call_ms * 1e3, 3),
            "launch": launch_desc}


def run_workload(name, dev, hbm_peak, peak_src):
    """A decode workload entry: REGIONS regions of at least REGION_MS of GPU time."""
    warm, calib = 3, 2
    run = DecodeRun(name, dev, extra_tokens=warm + calib + REGIONS * MAX_REGION_STEPS + 16, nstep_in=64)
    for i in range(warm):
        run.step(i)
    ms, _ = run.region(warm, calib)
    steps = max(1, min(MAX_REGION_STEPS, math.ceil(REGION_MS / (ms / calib))))
    first = warm + calib
    ctx0 = run.cache.len(0)
    regions = []
    with ClockSampler(dev.index) as clk:
        for r in range(REGIONS):
            ms, nbytes = run.region(first, steps)
            first += steps
            regions.append((ms, nbytes))
    ctx1 = run.cache.len(0)
    calls = steps * run.layers
    gbs = [b / (m * 1e-3) / 1e9 for m, b in regions]
    med = sorted(range(REGIONS), key=lambda r: gbs[r])[REGIONS // 2]
    ms_med, bytes_med = regions[med]
    entry = {
        "workload": name,
        "config": {"q_heads": run.Hq, "kv_heads": run.Hkv, "head_dim": D, "retrieval_kv_heads": run.nret, "S": S,
                   "W": W, "context": run.ctx, "batch": run.B, "layers": run.layers, "retrieval_kv": run.fmt},
        "gbs": round(gbs[med], 1),
        "us_per_token_layer": round(ms_med * 1e3 / calls, 3),
        "regions": dict(spread(gbs), unit="GB/s", steps_per_region=steps,
                        region_ms_median=round(ms_med, 2), context_range=[ctx0, ctx1]),
        "roofline": roofline_entry(name, bytes_med / calls, ms_med / calls, hbm_peak, peak_src, run.launch_desc),
        "clocks": clk.summary(),
        "gpu_launches": REGIONS * calls * run.lpl,
    }
    run.close()
    return entry


class PoolRun:
    """A pool workload: every sequence filled to its context on every layer (one seeded
    K/V draw per sequence, appended to each layer: the values do not change the work),
    then steps of duo_pool_decode_step over all sequences."""

    def __init__(self, name, dev, extra_tokens, nstep_in):
        import torch

        from head_split_kv_duo_b200 import inputs
        from head_split_kv_duo_b200.duo import DuoPool

        self.Hq, self.Hkv, self.nret, self.ctxs, self.layers, self.per_call = POOL_WORKLOADS[name]
        self.Hr, self.Hs = self.nret, self.Hkv - self.nret
        self.nseq = len(self.ctxs)
        pages = sum((c + extra_tokens + 127) // 128 + 1 for c in self.ctxs)
        mask = inputs.retrieval_mask(self.layers, self.Hkv, self.nret, seed=1)
        self.pool = DuoPool(self.layers, self.Hkv, mask, S, W, self.nseq, max(self.ctxs) + extra_tokens, pages,
                            q_heads=self.Hq, device=dev)
        self.seqs = [self.pool.open() for _ in self.ctxs]
        for i, c in enumerate(self.ctxs):
            k = inputs.randn((c, self.Hkv, D), 400 + 2 * i, device=dev)
            v = inputs.randn((c, self.Hkv, D), 401 + 2 * i, device=dev)
            for layer in range(self.layers):
                self.pool.append_kv(layer, self.seqs[i], k, v)
            del k, v
        torch.cuda.synchronize()
        self.nin = nstep_in
        self.qs = inputs.randn((nstep_in, self.layers, self.nseq, self.Hq, D), 17, device=dev)
        self.ks = inputs.randn((nstep_in, self.layers, self.nseq, self.Hkv, D), 18, device=dev)
        self.vs = inputs.randn((nstep_in, self.layers, self.nseq, self.Hkv, D), 19, device=dev)
        self.out = torch.empty(self.layers, self.nseq, self.Hq, D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(self.layers, self.nseq, self.Hq, dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream()

    def step(self, i, per_call=None):
        per_call = per_call or self.per_call
        j = i % self.nin
        nbytes = 0
        for l0 in range(0, self.layers, per_call):
            sl = slice(l0, l0 + per_call)
            for s in self.seqs:
                nbytes += per_call * decode_bytes(self.pool.len(s, l0) + 1, B=1, Hr=self.Hr, Hs=self.Hs, Hq=self.Hq)
            self.pool.decode_step(l0, per_call, self.seqs, self.qs[j, sl], self.ks[j, sl], self.vs[j, sl],
                                  out=self.out[sl], lse=self.lse[sl], stream=self.stream)
        return nbytes

    def region(self, first, steps, per_call=None):
        import torch
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(self.stream)
        nbytes = 0
        for i in range(first, first + steps):
            nbytes += self.step(i, per_call)
        t1.record(self.stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1), nbytes

    def close(self):
        import torch
        assert self.pool.device_status() == 0, "device status word set"
        self.pool.close()
        del self.pool, self.qs, self.ks, self.vs
        torch.cuda.empty_cache()


def run_pool_workload(name, dev, hbm_peak, peak_src):
    """A pool workload entry: REGIONS regions of at least REGION_MS, and the same steps
    with all layers in one decode_step call when the workload makes one call per layer."""
    warm, calib = 3, 2
    extra = warm + calib + 2 * REGIONS * MAX_REGION_STEPS + 16
    run = PoolRun(name, dev, extra, nstep_in=64)
    for i in range(warm):
        run.step(i)
    ms, _ = run.region(warm, calib)
    steps = max(1, min(MAX_REGION_STEPS, math.ceil(REGION_MS / (ms / calib))))
    first = warm + calib
    variants = [("per_call", run.per_call)] + ([("all_layers_one_call", run.layers)] if run.per_call < run.layers else [])
    res = {}
    with ClockSampler(dev.index) as clk:
        for vname, per_call in variants:
            regions = []
            for r in range(REGIONS):
                regions.append(run.region(first, steps, per_call))
                first += steps
            gbs = [b / (m * 1e-3) / 1e9 for m, b in regions]
            med = sorted(range(REGIONS), key=lambda r: gbs[r])[REGIONS // 2]
            calls = steps * (run.layers // per_call)
            ms_med, bytes_med = regions[med]
            res[vname] = {"layers_per_call": per_call, "gbs": round(gbs[med], 1),
                          "us_per_token_layer": round(ms_med * 1e3 / (steps * run.layers), 3),
                          "regions": dict(spread(gbs), unit="GB/s", steps_per_region=steps,
                                          region_ms_median=round(ms_med, 2)),
                          "roofline": roofline_entry(name, bytes_med / calls, ms_med / calls, hbm_peak, peak_src,
                                                     "pool append, then pool decode (all sequences, "
                                                     f"{per_call} layer(s) per launch)"),
                          "gpu_launches": REGIONS * calls * 2}
    entry = {"workload": name,
             "config": {"q_heads": run.Hq, "kv_heads": run.Hkv, "head_dim": D, "retrieval_kv_heads": run.nret, "S": S,
                        "W": W, "contexts": run.ctxs, "sequences": run.nseq, "layers": run.layers,
                        "retrieval_kv": "same (paged)"},
             "gbs": res["per_call"]["gbs"], "us_per_token_layer": res["per_call"]["us_per_token_layer"],
             "regions": res["per_call"]["regions"], "roofline": res["per_call"]["roofline"],
             "gpu_launches": res["per_call"]["gpu_launches"], "clocks": clk.summary()}
    if "all_layers_one_call" in res:
        entry["all_layers_one_call"] = res["all_layers_one_call"]
    run.close()
    return entry


def oracle_pool_sample(name, seconds, device="cpu"):
    """cpu_baseline of a pool workload: the oracle's decode of one layer of every
    sequence (each at its own context) until `seconds` of wall time (at least one)."""
    import numpy as np

    import oracle
    from head_split_kv_duo_b200 import inputs
    Hq, Hkv, nret, ctxs, layers, _ = POOL_WORKLOADS[name]
    mask = inputs.retrieval_mask(1, Hkv, nret, seed=1)[0].numpy().astype(bool)
    data = []
    for i, c in enumerate(ctxs):
        k = _u16(inputs.randn((1, c, Hkv, D), 400 + 2 * i, device=device).cpu())
        v = _u16(inputs.randn((1, c, Hkv, D), 401 + 2 * i, device=device).cpu())
        q = _u16(inputs.randn((1, 1, Hq, D), 17 + i, device=device).cpu())
        data.append((q, k, v, c))
    n, t_total, nbytes = 0, 0.0, 0
    while t_total < seconds or n == 0:
        t = time.perf_counter()
        for q, k, v, c in data:
            oracle.attend(q, k, v, mask, S, W, pos0=c - 1)
        t_total += time.perf_counter() - t
        nbytes += sum(decode_bytes(c, B=1, Hr=nret, Hs=Hkv - nret, Hq=Hq) for c in ctxs)
        n += 1
    return {"value": round(nbytes / t_total / 1e9, 3), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} oracle decode steps of one layer of all {len(ctxs)} sequences (contexts {ctxs}); "
                      f"{t_total:.1f} s wall on {oracle.num_threads()} threads", "seconds": round(t_total, 2)}


def run_headline(args, dev, dist, hbm_peak, peak_src):
    import torch
    K, warmup = args.steps, args.warmup
    extra = warmup + 2 + MAX_HEADLINE_REGIONS * K + 2 * K + 16
    run = DecodeRun(args.workload, dev, extra_tokens=extra, nstep_in=max(64, K), layers=args.layers)
    for i in range(warmup):
        run.step(i)
    # regions of exactly K steps: at least REGIONS, and until about HEADLINE_TOTAL_MS
    first = warmup
    regions = []
    with ClockSampler(dev.index) as clk:
        ms, nbytes = run.region(first, K, dist)
        first += K
        regions.append((ms, nbytes))
        nreg = max(REGIONS, min(MAX_HEADLINE_REGIONS, math.ceil(HEADLINE_TOTAL_MS / max(ms, 1e-3))))
        if dist:  # every rank times the same number of regions (the slowest rank's need)
            t = torch.tensor([nreg], device=dev, dtype=torch.int64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            nreg = int(t.item())
        for r in range(1, nreg):
            ms, nbytes = run.region(first, K, dist)
            first += K
            regions.append((ms, nbytes))
    reduced = [reduce_over_ranks(dist, m, b, dev) for m, b in regions]
    vals = [b / (m * 1e-3) / 1e9 for m, b in reduced]
    med = sorted(range(len(vals)), key=lambda r: vals[r])[len(vals) // 2]
    ms_max, bytes_sum = reduced[med]
    ms_own, bytes_own = regions[med]
    calls = K * run.layers
    # per-call durations for reference: one more region with an event pair around every call
    kev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), []]
    for i in range(first, first + K):
        run.step(i, kev)
    first += K
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in kev[2]]
    roof = roofline_entry(args.workload, bytes_own / calls, ms_own / calls, hbm_peak, peak_src, run.launch_desc)
    roof["event_bracketed_call_us"] = round(statistics.mean(dec_ms) * 1e3, 3)

    # ---- end-to-end through the public API with host buffers ----
    e2e = None
    if not args.skip_e2e:
        hq = run.qs[:K].cpu().pin_memory()
        hk = run.ks[:K].cpu().pin_memory()
        hv = run.vs[:K].cpu().pin_memory()
        hout = torch.empty(run.layers, run.B, run.Hq, D, dtype=torch.bfloat16).pin_memory()
        dq = torch.empty_like(run.qs[0])
        dk = torch.empty_like(run.ks[0])
        dv = torch.empty_like(run.vs[0])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eb = 0
        torch.cuda.synchronize()
        e0.record(run.stream)
        for i in range(K):
            dq.copy_(hq[i], non_blocking=True)
            dk.copy_(hk[i], non_blocking=True)
            dv.copy_(hv[i], non_blocking=True)
            for layer in range(run.layers):
                eb += run.nbytes_of(run.cache.len(layer) + 1)
                run.cache.append_decode(layer, dq[layer], dk[layer], dv[layer], out=run.out[layer],
                                        lse=run.lse[layer], stream=run.stream)
            hout.copy_(run.out, non_blocking=True)
        e1.record(run.stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        h2d = (dq.numel() + dk.numel() + dv.numel()) * 2
        e2e = {"value": round(eb / (ems * 1e-3) / 1e9, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * 2, "ms_per_step": round(ems / K, 4)}
    kv_gb = run.layers * run.nbytes_of(run.ctx) / 1e9
    head = {
        "value": round(vals[med], 1), "ms_per_step": round(ms_max / K, 4),
        "regions": dict(spread(vals), unit="GB/s", steps_per_region=K,
                        region_ms_median=round(ms_max, 2)),
        "config": {"workload": args.workload, "q_heads": run.Hq, "kv_heads": run.Hkv, "head_dim": D,
                   "retrieval_kv_heads": run.nret, "S": S, "W": W, "context": run.ctx, "batch": run.B,
                   "layers": run.layers, "retrieval_kv": run.fmt,
                   "l2": f"inputs larger than L2: {run.layers} layer caches of {kv_gb / run.layers:.2f} GB "
                         f"visited per step",
                   "parallelism": f"replicas{args.gpus}"},
        "dtype": "bf16" if run.fmt == "same" else f"bf16+{run.fmt}kv",
        "us_per_token_layer": round(ms_own * 1e3 / calls, 3),
        "roofline": roof,
        "gpu_launches": len(regions) * calls * run.lpl,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    run.close()
    return head


def run_prefill(args, dev, tc_peak, tc_sust, peak_src):
    L, C = args.prefill_len, args.prefill_chunk
    import torch

    from head_split_kv_duo_b200 import inputs
    from head_split_kv_duo_b200.duo import DuoCache

    mask = inputs.retrieval_mask(1, HKV, NRET, seed=1)
    k = inputs.randn((1, L, HKV, D), 200, device=dev)
    v = inputs.randn((1, L, HKV, D), 201, device=dev)
    q = inputs.randn((1, C, HQ, D), 202, device=dev)  # same queries for every chunk
    out = torch.empty_like(q)
    nchunks = L // C
    stream = torch.cuda.current_stream()

    def one():
        cache = DuoCache(1, HKV, D, mask, S, W, L, q_heads=HQ, dtype=torch.bfloat16, device=dev)
        evs = []
        for c in range(nchunks):
            sl = slice(c * C, (c + 1) * C)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            cache.prefill_chunk(0, q, k[:, sl], v[:, sl], out=out, want_lse=False, stream=stream)
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        cache.close()
        return sum(x.elapsed_time(y) for x, y in evs)

    for _ in range(args.prefill_warmup):
        one()
    with ClockSampler(dev.index) as clk:
        times = [one() for _ in range(args.prefill_steps)]
    fl = prefill_flops(L)
    tfl = [fl / (t * 1e-3) / 1e12 for t in times]
    ms = statistics.median(times)
    tflops = fl / (ms * 1e-3) / 1e12
    name = f"llama3-8b-gqa-prefill-{L // 1024}k-chunk{C // 1024}k"
    roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak,
            "peak_source": f"{peak_src} bf16_tflops (burst)", "unit": "TFLOP/s",
            "frac": round(tflops / tc_peak, 4), "frac_of_sustained": round(tflops / tc_sust, 4),
            "tensor_pipe_active": None, "traffic": None}
    rec = recorded_prefill_counters() if L == PREFILL_LEN and C == PREFILL_CHUNK else None
    if rec:
        roof["tensor_pipe_active"] = rec.get("tensor_pipe_active")
        roof["traffic"] = rec.get("dram_bytes_per_launch")
        roof["counters_source"] = rec.get("source")
    res = {"workload": name, "tflops": round(tflops, 1), "ms": round(ms, 2), "steps": args.prefill_steps,
           "runs": dict(spread(tfl), unit="TFLOP/s"), "algorithmic_tflop": round(fl / 1e12, 2),
           "roofline": roof, "clocks": clk.summary()}
    if not args.skip_cpu_baseline:
        res["cpu_baseline"] = oracle_prefill_sample(args, k.cpu(), v.cpu(), q.cpu(), mask, fl)
    return res


def run_gated(args, dev, tc_peak, tc_sust, peak_src):
    """Gated mixed attention of the identification phase on a Llama-3-8B-shaped layer
    (32 q / 8 kv heads, d 128, S 16, W 512) over one sequence of args.gated_len tokens."""
    import torch

    from head_split_kv_duo_b200 import inputs
    from head_split_kv_duo_b200.duo import gated_attention

    L = args.gated_len
    q = inputs.randn((1, L, HQ, D), 300, device=dev)
    k = inputs.randn((1, L, HKV, D), 301, device=dev)
    v = inputs.randn((1, L, HKV, D), 302, device=dev)
    alpha = torch.rand(HKV, generator=torch.Generator().manual_seed(3)).to(dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    times = []
    for i in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gated_attention(q, k, v, alpha, S, W, out=out, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    fl = gated_flops(L)
    tflops = fl / (ms * 1e-3) / 1e12
    return {"workload": f"llama3-8b-gqa-gated-{L // 1024}k", "tflops": round(tflops, 1), "ms": round(ms, 3),
            "steps": len(times), "runs": dict(spread([fl / (t * 1e-3) / 1e12 for t in times]), unit="TFLOP/s"),
            "algorithmic_tflop": round(fl / 1e12, 3),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst)", "unit": "TFLOP/s",
                         "frac": round(tflops / tc_peak, 4), "frac_of_sustained": round(tflops / tc_sust, 4)}}


# ---------------------------------------------------------- the oracle on the host

def _u16(t):
    import numpy as np
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleDecode:
    """The fp64 oracle's decode of one layer of a decode workload (the query of the
    newest token at position ctx - 1, every query head of every sequence).  INT4
    workloads go through the oracle's own quantiser and dequantiser, as the parity tests
    do; `ctx_cap` bounds the context of the sample.  Inputs are the seeded N(0,1) draws
    of the workload's first layer, drawn on `device` when given (faster) and copied to
    the host."""

    def __init__(self, name, ctx_cap=None, device="cpu"):
        import numpy as np

        import oracle
        from head_split_kv_duo_b200 import inputs

        self.oracle = oracle
        Hq, Hkv, nret, ctx, B, _, fmt = DECODE_WORKLOADS[name]
        self.ctx = min(ctx, ctx_cap) if ctx_cap else ctx
        self.B, self.Hq, self.Hkv, self.nret, self.fmt = B, Hq, Hkv, nret, fmt
        self.mask = inputs.retrieval_mask(1, Hkv, nret, seed=1)[0].numpy().astype(bool)
        k = inputs.randn((B, self.ctx, Hkv, D), 100, device=device).cpu()
        v = inputs.randn((B, self.ctx, Hkv, D), 101, device=device).cpu()
        self.q = _u16(inputs.randn((B, 1, Hq, D), 7, device=device).cpu())
        if fmt in ("int4", "fp8"):
            # fp64 K/V (the streaming heads' rows as they are); per retrieval head the codes
            # and scales from the oracle's quantiser, dequantised at every step
            self.k = k.float().numpy().astype(np.float64)
            self.v = v.float().numpy().astype(np.float64)
            quant = oracle.int4_quantize if fmt == "int4" else oracle.fp8_quantize
            self.codes = [(g, quant(_u16(k[:, :, g]).reshape(-1, D)), quant(_u16(v[:, :, g]).reshape(-1, D)))
                          for g in np.nonzero(self.mask)[0]]
        else:
            self.k, self.v = _u16(k), _u16(v)

    def step(self):
        if self.fmt in ("int4", "fp8"):
            deq = self.oracle.int4_dequantize if self.fmt == "int4" else self.oracle.fp8_dequantize
            for g, kc, vc in self.codes:
                self.k[:, :, g] = deq(*kc).reshape(self.B, self.ctx, D)
                self.v[:, :, g] = deq(*vc).reshape(self.B, self.ctx, D)
        return self.oracle.attend(self.q, self.k, self.v, self.mask, S, W, pos0=self.ctx - 1)

    def nbytes(self):
        return decode_bytes(self.ctx, B=self.B, Hr=self.nret, Hs=self.Hkv - self.nret, Hq=self.Hq, fmt=self.fmt)


def oracle_decode_sample(name, seconds, max_steps, ctx_cap=None, device="cpu"):
    """cpu_baseline of a decode workload: oracle decode steps of one layer until
    `seconds` of wall time (at least one)."""
    import oracle
    od = OracleDecode(name, ctx_cap, device)
    n, t_total = 0, 0.0
    while (t_total < seconds or n == 0) and n < max_steps:
        t = time.perf_counter()
        od.step()
        t_total += time.perf_counter() - t
        n += 1
    gbs = n * od.nbytes() / t_total / 1e9
    what = f"{n} oracle decode steps of one layer at context {od.ctx}"
    if od.ctx != DECODE_WORKLOADS[name][3]:
        what += f" (the workload's {DECODE_WORKLOADS[name][3]}-token context needs too much fp64 host memory)"
    if od.fmt in ("int4", "fp8"):
        what += f", each step dequantising the oracle's {od.fmt.upper()} codes of the retrieval heads, then attending"
    return {"value": round(gbs, 3), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{what}, batch {od.B}, all {od.Hq} query heads; {t_total:.1f} s wall on "
                      f"{oracle.num_threads()} threads", "seconds": round(t_total, 2), "steps": n}


def oracle_prefill_sample(args, k, v, q, mask, flops_total):
    """cpu_baseline of the pre-fill: the oracle on sampled query rows of every chunk (the
    first and last rows, rows around S and W, and random rows), all 32 query heads; the
    whole prompt's time is extrapolated by the count of visible (query, key) pairs."""
    import numpy as np

    import oracle
    L, C = args.prefill_len, args.prefill_chunk
    kb, vb, qb = _u16(k), _u16(v), _u16(q)
    m = mask[0].numpy().astype(bool)
    G = HQ // HKV
    rng = np.random.default_rng(0)
    nchunks = L // C
    per_chunk = {c: set([0, C - 1] + [x for x in (S - 1, S, S + 1, W - 1, W, W + 1) if 0 <= x < C])
                 for c in range(nchunks)}
    for r in rng.integers(0, L, args.prefill_oracle_rows):
        per_chunk[int(r) // C].add(int(r) % C)
    pairs_sample, t_total, nrows = 0, 0.0, 0
    for c in range(nchunks):
        rows = sorted(per_chunk[c])
        ids = [r * HQ + h for r in rows for h in range(HQ)]
        t = time.perf_counter()
        oracle.attend(qb, kb[:, :(c + 1) * C], vb[:, :(c + 1) * C], m, S, W, pos0=c * C, rows=ids)
        t_total += time.perf_counter() - t
        nrows += len(ids)
        for r in rows:
            i = c * C + r
            pairs_sample += sum(visible_pairs(i, m[h // G]) for h in range(HQ))
    pairs_total = flops_total // (4 * D)
    est_s = t_total * pairs_total / pairs_sample
    return {"value": round(flops_total / est_s / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "extrapolated": True, "seconds_sampled": round(t_total, 2),
            "seconds_extrapolated": round(est_s, 1),
            "sample": f"{nrows} (query row, head) pairs of the {L // 1024}K prompt ({pairs_sample} of the "
                      f"{pairs_total} visible (query, key) pairs), {t_total:.1f} s wall on "
                      f"{oracle.num_threads()} threads; time extrapolated by visible-pair count"}


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(DECODE_WORKLOADS))
    ap.add_argument("--layers", type=int, default=0,
                    help="layer caches of the headline workload (0: the model's 32); small profiling captures only")
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workloads", default="all",
                    help="comma-separated decode workloads for the 'workloads' entries, 'all' or 'none'")
    ap.add_argument("--skip-prefill", action="store_true")
    ap.add_argument("--skip-decode", action="store_true", help="time only the pre-fill workload")
    ap.add_argument("--prefill-len", type=int, default=PREFILL_LEN)
    ap.add_argument("--prefill-chunk", type=int, default=PREFILL_CHUNK)
    ap.add_argument("--prefill-steps", type=int, default=5)
    ap.add_argument("--prefill-warmup", type=int, default=1)
    ap.add_argument("--prefill-oracle-rows", type=int, default=256)
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-gated", action="store_true", help="skip the gated (identification-phase) forward")
    ap.add_argument("--gated-len", type=int, default=32768)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-seconds", type=float, default=4.0)
    ap.add_argument("--oracle-max-steps", type=int, default=40)
    ap.add_argument("--ref-layers", type=int, default=4,
                    help="reference arm: layers of the headline step the oracle decodes per step")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args)

    import torch
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()
    if args.skip_decode:
        if rank == 0:
            res = {"prefill": run_prefill(args, dev, tc_peak, tc_sust, peak_src)}
            if not args.skip_gated:
                res["gated"] = run_gated(args, dev, tc_peak, tc_sust, peak_src)
            print(json.dumps(res))
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    head = run_headline(args, dev, dist, hbm_peak, peak_src)
    res = {"metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic", "config": head["config"],
           "us_per_token_layer": head["us_per_token_layer"], "regions": head["regions"],
           "roofline": head["roofline"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
           "e2e": head["e2e"]}
    # the remaining configurations run on rank 0 only (each rank is an independent replica)
    if rank == 0:
        if args.workloads != "none":
            names = sorted(DECODE_WORKLOADS) + sorted(POOL_WORKLOADS) if args.workloads == "all" \
                else args.workloads.split(",")
            res["workloads"] = {}
            for name in names:
                if name in POOL_WORKLOADS:
                    e = run_pool_workload(name, dev, hbm_peak, peak_src)
                    if not args.skip_cpu_baseline:
                        e["cpu_baseline"] = oracle_pool_sample(name, args.oracle_seconds, dev)
                else:
                    e = run_workload(name, dev, hbm_peak, peak_src)
                    if not args.skip_cpu_baseline:
                        cap = 1 << 17 if DECODE_WORKLOADS[name][6] == "int4" else None
                        e["cpu_baseline"] = oracle_decode_sample(name, args.oracle_seconds, args.oracle_max_steps,
                                                                 cap, dev)
                res["workloads"][name] = e
        if not args.skip_prefill:
            res["prefill"] = run_prefill(args, dev, tc_peak, tc_sust, peak_src)
        if not args.skip_gated:
            res["gated"] = run_gated(args, dev, tc_peak, tc_sust, peak_src)
        if not args.skip_cpu_baseline:
            res["cpu_baseline"] = oracle_decode_sample(args.workload, args.oracle_seconds, args.oracle_max_steps,
                                                       device=dev)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores, W warm-up steps then K
    timed steps; a step is the oracle's decode of `ref_layers` layers of the headline
    step (one layer's seeded K/V stands in for each of them: the oracle's time does not
    depend on the values)."""
    import oracle
    t_wall = time.perf_counter()
    od = OracleDecode(args.workload, 1 << 17 if DECODE_WORKLOADS[args.workload][6] == "int4" else None)
    for _ in range(args.warmup):
        for _ in range(args.ref_layers):
            od.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for _ in range(args.ref_layers):
            od.step()
    secs = time.perf_counter() - t0
    nbytes = args.steps * args.ref_layers * od.nbytes()
    gbs = nbytes / secs / 1e9
    Hq, Hkv, nret, ctx, B, layers, fmt = DECODE_WORKLOADS[args.workload]
    cb = {"value": round(gbs, 3), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
          "sample": f"{args.steps} steps, each the oracle's decode of {args.ref_layers} of the {layers} layers of "
                    f"the step at context {od.ctx}; {secs:.1f} s wall on {oracle.num_threads()} threads"}
    res = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3 / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": args.workload, "q_heads": Hq, "kv_heads": Hkv, "head_dim": D,
                      "retrieval_kv_heads": nret, "S": S, "W": W, "context": ctx, "batch": B, "layers": layers,
                      "retrieval_kv": fmt},
           "cpu_baseline": cb,
           "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "wall_s": round(time.perf_counter() - t_wall, 1)}
    print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
