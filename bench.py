#!/usr/bin/env python
"""Benchmark of the hybrid-head KV attention path on B200.

Headline workload (N = 1): decode attention of a Llama-3-8B-shaped GQA layer (32 q /
8 kv heads, d 128, 4 retrieval + 4 streaming kv heads, S 16, W 512, bf16) at a
128K-token context, batch 1.  One step = for each of 4 layer caches in turn (4 x
1.08 GB of K/V, larger than L2, so no L2 flush is needed): append the new token's
K/V and run decode attention -- the whole decode path (append/evict, retrieval
split-KV, streaming sink+ring, merge).  value = algorithmic HBM bytes of the decode
attention per step / step time (GB/s), the step timed with no events between its
launches; each append + attend goes through duo_append_decode (one fused launch at
batch 1).  roofline.achieved divides the same bytes by the timed region's time per
decode call; a second pass of the same steps with an event pair around every call
gives event_bracketed_call_us for reference; roofline.traffic is the DRAM traffic per
launch from the committed ncu capture, reported while the sources of the workload's
kernels still hash to the recorded value.  The chunked pre-fill workload (256K
prompt in 32K chunks, same shape) is timed after it and reported under "prefill",
and the identification-phase gated forward (32K tokens) under "gated".

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of
the same workload (the reference arm).  Under torchrun every rank runs an
independent replica (the path does not shard); value sums the ranks' bytes over
the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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
ROT_LAYERS = 4
PREFILL_LEN, PREFILL_CHUNK = 262144, 32768

# decode workloads: (q heads, kv heads, retrieval kv heads, context, batch, layers, retrieval format);
# `layers` caches are visited in turn each step (the headline rotates 4 so that a step
# touches more K/V than L2 holds; the INT4 stack is the 32-layer model itself)
DECODE_WORKLOADS = {
    "llama3-8b-gqa-decode-128k-b1": (32, 8, 4, 131072, 1, 4, "same"),
    "llama3-8b-gqa-decode-128k-b4": (32, 8, 4, 131072, 4, 2, "same"),
    "llama2-7b-mha-decode-32k-b1": (32, 32, 8, 32768, 1, 8, "same"),
    "llama2-7b-mha-decode-32k-b8": (32, 32, 8, 32768, 8, 2, "same"),
    "llama3-8b-gqa-decode-1m-int4-32l": (32, 8, 4, 1 << 20, 1, 32, "int4"),
}


def decode_bytes(len_, B=1, Hr=NRET, Hs=HKV - NRET, Hq=HQ, d=D, fmt="same"):
    """Algorithmic HBM bytes of one decode-attention call: every visible K and V row
    once (bf16 rows, or INT4 codes plus fp16 scale/zero), the queries, the outputs and
    the lse."""
    kv = 2 * d * 2
    rkv = 2 * (d // 2 + 4) if fmt == "int4" else kv
    return B * (Hr * len_ * rkv + Hs * min(len_, S + W) * kv) + B * Hq * d * 2 * 2 + B * Hq * 4


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


def kernel_hash(workload):
    """Hash of the sources of the decode kernels a workload runs: recorded DRAM traffic
    is void once they change."""
    files = ["k_decode_tc.cu", "tcgen05.cuh", "decode_merge.cuh", "device_common.cuh", "duo_internal.h"]
    if "int4" in workload:
        files.append("k_decode_int4_tc.cu")
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "head_split_kv_duo_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes (read + write) per decode launch from the committed ncu summary of
    this workload, when it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(workload)
    if not rec or rec.get("kernel_hash") != kernel_hash(workload):
        return None
    return rec.get("dram_bytes_per_launch")


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


def run_ours(args, rank, world, dist):
    import torch

    from head_split_kv_duo_b200 import inputs
    from head_split_kv_duo_b200.duo import DuoCache

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()
    steps, warmup = args.steps, args.warmup
    Hq, Hkv, nret, ctx, B, nlayers, fmt = DECODE_WORKLOADS[args.workload]
    if args.layers:
        nlayers = args.layers
    Hr, Hs = nret, Hkv - nret
    max_len = ctx + warmup + 3 * steps + 16  # warm-up, timed and event passes, e2e pass
    mask = inputs.retrieval_mask(nlayers, Hkv, nret, seed=1)
    cache = DuoCache(nlayers, Hkv, D, mask, S, W, max_len, batch=B, q_heads=Hq, dtype=torch.bfloat16,
                     retr_fmt=fmt, device=dev)
    # fill each layer to `ctx` tokens (seeded N(0,1) K/V), in pieces of at most 2^18 tokens
    piece = min(ctx, 1 << 18)
    for layer in range(nlayers):
        for t0 in range(0, ctx, piece):
            n = min(piece, ctx - t0)
            k = inputs.randn((B, n, Hkv, D), 100 + 1000 * layer + 2 * t0 // piece, device=dev)
            v = inputs.randn((B, n, Hkv, D), 101 + 1000 * layer + 2 * t0 // piece, device=dev)
            cache.append_kv(layer, k, v)
            del k, v
    torch.cuda.synchronize()
    # per-step inputs: q, k, v of the new token for every layer
    nstep_in = warmup + 2 * steps
    qs = inputs.randn((nstep_in, nlayers, B, Hq, D), 7, device=dev)
    ks = inputs.randn((nstep_in, nlayers, B, 1, Hkv, D), 8, device=dev)
    vs = inputs.randn((nstep_in, nlayers, B, 1, Hkv, D), 9, device=dev)
    out = torch.empty(nlayers, B, Hq, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(nlayers, B, Hq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def nbytes_of(n):
        return decode_bytes(n, B=B, Hr=Hr, Hs=Hs, Hq=Hq, fmt=fmt)

    def step(i, ev=None):
        nbytes = 0
        for layer in range(nlayers):
            n = cache.len(layer) + 1
            if ev is not None:
                ev[0].record(stream)
            # append the step's token and attend: one launch on the bf16 tcgen05 path
            cache.append_decode(layer, qs[i, layer], ks[i, layer], vs[i, layer], out=out[layer], lse=lse[layer],
                                stream=stream)
            if ev is not None:
                ev[1].record(stream)
                ev[2].append((ev[0], ev[1]))
                ev[0] = torch.cuda.Event(enable_timing=True)
                ev[1] = torch.cuda.Event(enable_timing=True)
            nbytes += nbytes_of(n)
        return nbytes

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    # timed region: the steps alone (no events between launches)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nbytes = 0
    with ClockSampler(dev.index) as clk:
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(warmup, warmup + steps):
            nbytes += step(i)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    # per-call durations of the decode call for the roofline: the same steps again, with
    # an event pair around every call (the events add a little time between launches)
    kev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), []]
    for i in range(warmup + steps, warmup + 2 * steps):
        step(i, kev)
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in kev[2]]
    assert cache.device_status() == 0, "device status word set"
    ms_max, bytes_sum = reduce_over_ranks(dist, ms, nbytes, dev)
    value = bytes_sum / (ms_max * 1e-3) / 1e9
    us_per_token_layer = ms * 1e3 / (steps * nlayers)
    dec_avg_ms = statistics.mean(dec_ms)
    per_launch_bytes = nbytes / (steps * nlayers)
    # the decode call's duration over the timed region: every launch in it belongs to a
    # decode call (one fused launch at batch 1), so this includes the gaps between them
    call_ms = ms / (steps * nlayers)
    achieved = per_launch_bytes / (call_ms * 1e-3) / 1e9

    # ---- end-to-end through the public API with host buffers ----
    e2e = None
    if not args.skip_e2e:
        hq = qs.cpu().pin_memory()
        hk = ks.cpu().pin_memory()
        hv = vs.cpu().pin_memory()
        hout = torch.empty(nlayers, B, Hq, D, dtype=torch.bfloat16).pin_memory()
        dq = torch.empty_like(qs[0])
        dk = torch.empty_like(ks[0])
        dv = torch.empty_like(vs[0])
        # lengths cannot be rewound: this pass keeps appending (max_len has room for it)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        eb = 0
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(warmup, warmup + steps):
            dq.copy_(hq[i], non_blocking=True)
            dk.copy_(hk[i], non_blocking=True)
            dv.copy_(hv[i], non_blocking=True)
            for layer in range(nlayers):
                eb += nbytes_of(cache.len(layer) + 1)
                cache.append_decode(layer, dq[layer], dk[layer], dv[layer], out=out[layer], lse=lse[layer],
                                    stream=stream)
            hout.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        h2d = (dq.numel() + dk.numel() + dv.numel()) * 2
        e2e = {"value": round(eb / (ems * 1e-3) / 1e9, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * 2, "ms_per_step": round(ems / steps, 4)}
    cache.close()
    del cache
    torch.cuda.empty_cache()

    # ---- chunked pre-fill (Llama-3-8B GQA, 256K in 32K chunks) ----
    prefill = None
    if not args.skip_prefill:
        prefill = run_prefill(args, dev, tc_peak, tc_sust, peak_src)
    gated = None
    if not args.skip_gated:
        gated = run_gated(args, dev, tc_peak, tc_sust, peak_src)

    kv_gb = nlayers * nbytes_of(ctx) / 1e9
    # per layer and step: one fused append + decode launch (bf16, batch 1), else the append
    # then the decode; an INT4 layer decodes its bf16 streaming heads and its INT4
    # retrieval heads in two launches
    if fmt == "same":
        launches_per_layer, launch_desc = (1, "fused append+decode") if B == 1 else (2, "append, then decode")
    else:
        launches_per_layer = 3 if Hkv > nret else 2
        launch_desc = "append, bf16 streaming-head decode, INT4 retrieval-head decode"
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(ms_max / steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if fmt == "same" else "bf16+int4kv", "data": "synthetic",
        "config": {"workload": args.workload, "q_heads": Hq, "kv_heads": Hkv, "head_dim": D, "retrieval_kv_heads": nret,
                   "S": S, "W": W, "context": ctx, "batch": B, "layers": nlayers, "retrieval_kv": fmt,
                   "l2": f"inputs larger than L2: {nlayers} layer caches of {kv_gb / nlayers:.2f} GB visited per step",
                   "parallelism": f"replicas{world}"},
        "us_per_token_layer": round(us_per_token_layer, 3),
        "roofline": {"bound": "hbm", "kernel": "decode", "achieved": round(achieved, 1),
                     "peak": hbm_peak, "peak_source": f"{peak_src} hbm_gbs (burst copy)", "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "frac_of_8tbs_spec": round(achieved / 8000.0, 4),
                     "traffic": recorded_traffic(args.workload),
                     "algorithmic_bytes_per_launch": int(per_launch_bytes), "avg_launch_us": round(call_ms * 1e3, 3),
                     "event_bracketed_call_us": round(dec_avg_ms * 1e3, 3),
                     "launch": launch_desc},
        "gpu_launches": steps * nlayers * launches_per_layer,
        "clocks": clk.summary(),
        "e2e": e2e,
        "prefill": prefill,
        "gated": gated,
    }
    return res


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
    times = [one() for _ in range(args.prefill_steps)]
    ms = statistics.mean(times)
    fl = prefill_flops(L)
    tflops = fl / (ms * 1e-3) / 1e12
    name = f"llama3-8b-gqa-prefill-{L // 1024}k-chunk{C // 1024}k"
    return {"workload": name, "tflops": round(tflops, 1), "ms": round(ms, 2),
            "steps": args.prefill_steps, "algorithmic_tflop": round(fl / 1e12, 2),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst)", "unit": "TFLOP/s",
                         "frac": round(tflops / tc_peak, 4), "frac_of_sustained": round(tflops / tc_sust, 4)}}


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
    for i in range(4):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        gated_attention(q, k, v, alpha, S, W, out=out, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            times.append(a.elapsed_time(b))
    ms = statistics.mean(times)
    fl = gated_flops(L)
    tflops = fl / (ms * 1e-3) / 1e12
    return {"workload": f"llama3-8b-gqa-gated-{L // 1024}k", "tflops": round(tflops, 1), "ms": round(ms, 3),
            "steps": len(times), "algorithmic_tflop": round(fl / 1e12, 3),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst)", "unit": "TFLOP/s",
                         "frac": round(tflops / tc_peak, 4), "frac_of_sustained": round(tflops / tc_sust, 4)}}


# ---------------------------------------------------------- reference arm

def oracle_sample(args):
    """Time the fp64 oracle on decode steps of the headline workload (one layer at
    128K context; each step = one query token, all 32 query heads)."""
    import numpy as np
    import torch

    import oracle
    from head_split_kv_duo_b200 import inputs

    mask = inputs.retrieval_mask(1, HKV, NRET, seed=1)[0].numpy().astype(bool)
    k = inputs.randn((1, CTX, HKV, D), 100).view(torch.int16).numpy().view(np.uint16)
    v = inputs.randn((1, CTX, HKV, D), 101).view(torch.int16).numpy().view(np.uint16)
    q = inputs.randn((1, 1, HQ, D), 7).view(torch.int16).numpy().view(np.uint16)
    oracle.attend(q, k[:, :1024], v[:, :1024], mask, S, W, pos0=1023)  # load / warm
    n, t_total = 0, 0.0
    budget = args.oracle_seconds
    while t_total < budget and n < args.oracle_max_steps:
        t = time.perf_counter()
        oracle.attend(q, k, v, mask, S, W, pos0=CTX - 1)
        t_total += time.perf_counter() - t
        n += 1
    gbs = n * decode_bytes(CTX) / t_total / 1e9
    return {"value": round(gbs, 3), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} decode steps of one layer at context {CTX} (all 32 query heads), "
                      f"{t_total:.1f} s wall on {oracle.num_threads()} threads",
            "seconds": round(t_total, 2), "steps": n}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(DECODE_WORKLOADS))
    ap.add_argument("--layers", type=int, default=0,
                    help="layer caches to rotate through instead of the workload's (small profiling captures)")
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-prefill", action="store_true")
    ap.add_argument("--skip-decode", action="store_true", help="time only the pre-fill workload")
    ap.add_argument("--prefill-len", type=int, default=PREFILL_LEN)
    ap.add_argument("--prefill-chunk", type=int, default=PREFILL_CHUNK)
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-gated", action="store_true", help="skip the gated (identification-phase) forward")
    ap.add_argument("--gated-len", type=int, default=32768)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-steps", type=int, default=2)
    ap.add_argument("--prefill-warmup", type=int, default=1)
    ap.add_argument("--oracle-seconds", type=float, default=6.0)
    ap.add_argument("--oracle-max-steps", type=int, default=40)
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        t0 = time.perf_counter()
        for _ in range(args.warmup):
            pass
        cb = oracle_sample(args)
        res = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s", "n_gpus": args.gpus,
               "steps": cb["steps"], "warmup": args.warmup, "ms_per_step": round(cb["seconds"] * 1e3 / max(cb["steps"], 1), 3),
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": {"workload": WORKLOAD, "q_heads": HQ, "kv_heads": HKV, "head_dim": D,
                          "retrieval_kv_heads": NRET, "S": S, "W": W, "context": CTX, "batch": 1},
               "cpu_baseline": cb,
               "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
               "wall_s": round(time.perf_counter() - t0, 1)}
        print(json.dumps(res))
        return 0

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    if args.skip_decode:
        import torch
        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
        torch.cuda.set_device(dev)
        _, tc_peak, tc_sust, src = peaks()
        if rank == 0:
            res = {"prefill": run_prefill(args, dev, tc_peak, tc_sust, src)}
            if not args.skip_gated:
                res["gated"] = run_gated(args, dev, tc_peak, tc_sust, src)
            print(json.dumps(res))
        return 0
    res = run_ours(args, rank, world, dist)
    if rank == 0 and not args.skip_cpu_baseline:
        res["cpu_baseline"] = oracle_sample(args)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))
    return 0


if __name__ == "__main__":
    sys.exit(main())
