#!/usr/bin/env python
"""Decode throughput of one OPT layer block with 4-bit weights and a 4-bit KV cache.

Default workload (one GPU): the OPT-6.7B-shaped layer -- hidden 4096, 32 heads x 128,
FFN 16384 -- over a zig-zag block of 8 GPU batches x 64 sequences, prompt 512 (prefilled,
untimed), then decode steps at positions 512, 513, ...  A step is one fg_layer_decode
over the whole block: LN1, QKV W4A16 GEMM, 4-bit KV append, decode attention over the
4-bit cache, out-proj GEMM + residual, LN2, FC1 GEMM + ReLU, FC2 GEMM + residual.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload ...]

With N > 1 (launched by torch.distributed.run) every rank runs its own block of
sequences (independent replicas, weak scaling, no collective on the data path); the
timed region is bracketed by barriers and the time is the max over ranks.
The reference arm (--impl reference) times the CPU oracle on a bounded sample of the
same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "opt-6.7b-layer": dict(hidden=4096, heads=32, ffn=16384, nb=8, gbs=64, prompt=512, steps=32),
    "opt-125m-layer": dict(hidden=768, heads=12, ffn=3072, nb=1, gbs=4, prompt=32, steps=8),
    # the same OPT-6.7B-shaped block with the layer's products in the W4A8 form (int8 activations,
    # one scale per row; two-level 4-bit weights; the KV cache unchanged)
    "opt-6.7b-layer-w4a8": dict(hidden=4096, heads=32, ffn=16384, nb=8, gbs=64, prompt=512, steps=32, act_bits=8),
    # prompt processing of the OPT-6.7B-shaped block: one prefill of 512 tokens for each of the
    # 512 sequences through one layer (the cache filled from position 0)
    "opt-6.7b-prefill": dict(hidden=4096, heads=32, ffn=16384, nb=8, gbs=64, prompt=512, steps=32, phase="prefill"),
    "opt-6.7b-prefill-w4a8": dict(hidden=4096, heads=32, ffn=16384, nb=8, gbs=64, prompt=512, steps=32,
                                  phase="prefill", act_bits=8),
    # OPT-30B-shaped stack: 48 layers whose W4 blobs stay in pinned host memory and are
    # prefetched layer by layer on a side stream; KV4 caches resident in HBM
    "opt-30b-stack": dict(hidden=7168, heads=56, ffn=28672, nb=4, gbs=64, prompt=512, steps=32, layers=48),
    "opt-30b-stack-w4a8": dict(hidden=7168, heads=56, ffn=28672, nb=4, gbs=64, prompt=512, steps=32, layers=48,
                               act_bits=8),
    # OPT-175B-shaped stack: weights AND KV4 caches in pinned host memory; each layer's cache is
    # filled into a device staging cache before the layer and its new slots written back after.
    # The model has 96 layers (about 3.06 GB of host memory each); unless --layers is given the
    # run takes at most 16, and no more than half the host's available memory holds, every
    # layer with its own host buffers.
    "opt-175b-stack": dict(hidden=12288, heads=96, ffn=49152, nb=8, gbs=32, prompt=512, steps=32, layers=16,
                           model_layers=96, kv_host=True),
}
METRIC = "decode tokens/s per OPT layer block (W4 KV4)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], tc_burst=d["bf16_tflops"], tc_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, tc_burst=1590.0, tc_sustained=1400.0, source="fallback")


def kernel_work(wl, S, L_avg, group=64, fused_append=True):
    """Algorithmic work per launch of each kernel of one step (bytes or flops).  Decode rows
    append their k, v inside the attention kernel (fused_append); prompt rows append apart.
    W4A8 layers: the products are int8 ("tensor_i8") and each takes its input from an activation
    quantiser (fp16 in, int8 and a row scale out)."""
    h, F, H = wl["hidden"], wl["ffn"], wl["heads"]
    gemm = "tensor_i8" if wl.get("act_bits") == 8 else "tensor"
    act8 = lambda k: ("hbm", S * k * 3 + S * 4)
    d = h // H
    kv_tok = 2 * (d // 2 + 4 * (d // group))         # K and V codes + fp16 min/scale per (seq, head, token)
    w4 = lambda n, k: n * k // 2 + n * (k // group) * 4  # packed weight bytes
    return {
        "ln1": ("hbm", 2 * S * h * 2 + 4 * h),
        "qkv_gemm": (gemm, 2 * S * 3 * h * h),
        "kv_append": ("hbm", S * 2 * h * 2 + S * H * kv_tok),  # fp16 k, v in; codes and metadata out
        # decode attention appends the step's k, v itself: fp16 q, k, v in, o out, the new
        # codes and metadata written, the cache read up to and including them
        "attention": ("hbm", S * H * L_avg * kv_tok + 2 * S * h * 2
                      + ((2 * S * h * 2 + S * H * kv_tok) if fused_append else 0)),
        "out_gemm": (gemm, 2 * S * h * h),
        "ln2": ("hbm", 2 * S * h * 2 + 4 * h),
        "fc1_gemm": (gemm, 2 * S * F * h),
        "fc2_gemm": (gemm, 2 * S * h * F),
        "qkv_act8": act8(h), "out_act8": act8(h), "fc1_act8": act8(h), "fc2_act8": act8(F),
    }, {"w4_bytes": w4(3 * h, h) + w4(h, h) + w4(F, h) + w4(h, F), "kv_bytes_per_token": kv_tok}


def kernel_units(wl, S, L_avg):
    """Units one launch of each kernel processes, the scale for traffic taken on a smaller case."""
    h, F, H = wl["hidden"], wl["ffn"], wl["heads"]
    return {"ln1": S, "qkv_gemm": S, "kv_append": S, "attention": S * H * L_avg, "out_gemm": S, "ln2": S,
            "fc1_gemm": S, "fc2_gemm": S, "qkv_act8": S, "out_act8": S, "fc1_act8": S, "fc2_act8": S}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows]
        reasons = set()
        for r in rows:
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(rows),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------------
# CPU oracle baseline (test infrastructure; only this leg of the benchmark loads it)
# ----------------------------------------------------------------------------------------

class OracleSample:
    """One oracle decode step for `n_seqs` sequences at position `prompt`.

    Set-up (untimed): the layer's seeded fp16 weights quantised by the oracle, and the
    sampled sequences' caches filled with `prompt` tokens of seeded N(0,1) k/v in 4-bit
    form (the decode step's work does not depend on how they were produced).
    step() times oracle.layer_rows as it stands (it dequantises the weights, then runs
    the rows on `threads` threads)."""

    def __init__(self, wl, n_seqs: int, threads: int, seed: int = 0):
        import oracle
        import seeded_inputs as si
        self.oracle = oracle
        h, H, F, P = wl["hidden"], wl["heads"], wl["ffn"], wl["prompt"]
        self.H, self.P, self.n, self.threads = H, P, n_seqs, threads
        maxL = (P + wl["steps"] + 63) // 64 * 64
        self.w4a8 = wl.get("act_bits") == 8
        w16 = si.layer_weights_f16(seed, h, F)
        self.W = oracle.W4A8LayerWeights(w16) if self.w4a8 else oracle.LayerWeights(w16)
        self.cache = oracle.KVCache(n_seqs, H, h // H, maxL)
        for s in range(n_seqs):
            k = si.normal_f16(seed, si.STREAM["k_new"], (P, h), 1.0, start=s * P * h)
            v = si.normal_f16(seed, si.STREAM["v_new"], (P, h), 1.0, start=s * P * h)
            oracle.kv_append(self.cache, k, v, np.full(P, s), np.arange(P))
        self.x = si.decode_inputs(seed, 0, n_seqs, h)

    def step(self) -> float:
        t0 = time.perf_counter()
        run = self.oracle.layer_rows_w4a8 if self.w4a8 else self.oracle.layer_rows
        run(self.W, self.H, self.cache, self.x, np.arange(self.n), np.full(self.n, self.P), nthreads=self.threads)
        return time.perf_counter() - t0


def oracle_quant_baseline(kind: str, group: int, log2_elems: int, bits: int = 4):
    """The oracle's quantise (or dequantise) on the quantize-sweep recipe, timed on this host:
    one thread, then the rows split over every host thread (the oracle's C loops release the
    GIL).  A bounded sample of min(2^log2_elems, 2^26) elements stands in for the full tensor;
    the oracle's time per element does not depend on the tensor's size."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    import seeded_inputs as si
    n = 1 << min(log2_elems, 26)
    x = si.sweep_tensor(0, n, group=group)
    rows = x.shape[0]
    packed = oracle.quantize(x, group=group, bits=bits) if kind == "dequantize" else None

    def work(lo, hi):
        if kind == "quantize":
            oracle.quantize(x[lo:hi], group=group, bits=bits)
        else:
            q = oracle.Packed(packed.codes[lo:hi], packed.mins[lo:hi], packed.scales[lo:hi],
                              (hi - lo, x.shape[1]), 1, group, bits)
            oracle.dequantize(q)

    bytes_ = n * (2 + bits / 8 + 4.0 / group)
    t0 = time.perf_counter()
    work(0, rows)
    t1 = time.perf_counter() - t0
    threads = os.cpu_count() or 1
    parts = [(rows * i // threads, rows * (i + 1) // threads) for i in range(threads)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        t0 = time.perf_counter()
        list(ex.map(lambda p: work(*p), parts))
        tn = time.perf_counter() - t0
    return {"value": bytes_ / tn / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"oracle {kind} of 2^{min(log2_elems, 26)} elements of the sweep recipe, rows split over "
                      f"{threads} threads",
            "single_thread": {"value": bytes_ / t1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"the same 2^{min(log2_elems, 26)} elements, one thread"}}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # one sampled sequence per host thread (the oracle splits a step's rows by sequence)
    n_seqs = max(1, min(os.cpu_count() or 1, 32, wl["nb"] * wl["gbs"]))
    threads = n_seqs
    sample = OracleSample(wl, n_seqs, threads)
    times = []
    for i in range(args.warmup + args.steps):
        t = sample.step()
        if i >= args.warmup:
            times.append(t)
    mean = sum(times) / len(times)
    value = n_seqs / mean
    S = wl["nb"] * wl["gbs"]
    desc = (f"{n_seqs} of {S} sequences, one decode step at position {wl['prompt']} per step "
            f"(cache of {wl['prompt']} tokens); {threads} threads")
    t1 = OracleSample(wl, 1, 1).step()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "block": f"{wl['nb']}x{wl['gbs']}", "hidden": wl["hidden"],
                   "prompt": wl["prompt"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc,
                         "single_thread": {"value": 1.0 / t1, "unit": "tokens/s", "cores": 1,
                                           "sample": f"1 of {S} sequences, one decode step, one thread"}},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------------------
# GPU path
# ----------------------------------------------------------------------------------------

def read_traffic(kernel: str, workload: str, units: float):
    """Per-launch DRAM bytes (read + write) from a committed ncu capture, if it was taken on the
    current source of the kernel.  A capture of a smaller case is scaled by the units one launch
    processes (for attention: sequence x head x context-token triples), the kernel's traffic
    being proportional to them."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e:
        return None
    import hashlib
    src = os.path.join(ROOT, "bit_compressed_decode_b200", "csrc", e["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != e["source_sha"]:
            return None
    return round(e["dram_bytes_per_launch"] * units / e["units_per_launch"])


def run_e2e(torch, fg, step, stream, dev, xs, S, h, P, nsteps_cfg, steps, warmup, barrier):
    """Milliseconds for `steps` decode steps with host inputs and outputs: step i's hidden states
    and positions are copied H2D from pinned memory and its output D2H into pinned memory, inside
    the timed region.  The copies run on their own stream into / out of two device buffers each,
    ordered by events: H2D(i+1) waits until step i-1 has read that buffer, step i waits for
    H2D(i) and for D2H(i-2) to have drained its output buffer, D2H(i) waits for step i."""
    xh = [torch.empty((S, h), dtype=torch.float16, pin_memory=True) for _ in range(2)]
    for i in range(2):
        xh[i].copy_(xs[i])
    ph = [torch.full((S,), P + t, dtype=torch.int32).pin_memory() for t in range(nsteps_cfg)]
    oh = [torch.empty((S, h), dtype=torch.float16, pin_memory=True) for _ in range(2)]
    xd = [torch.empty((S, h), dtype=torch.float16, device=dev) for _ in range(2)]
    pd = [torch.empty((S,), dtype=torch.int32, device=dev) for _ in range(2)]
    od = [torch.empty((S, h), dtype=torch.float16, device=dev) for _ in range(2)]
    cp = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    h2d_done = [ev(), ev()]
    comp_done = [ev(), ev()]
    d2h_done = [ev(), ev()]

    def h2d(i):
        b = i % 2
        with torch.cuda.stream(cp):
            xd[b].copy_(xh[i % 2], non_blocking=True)
            pd[b].copy_(ph[(warmup + i) % nsteps_cfg], non_blocking=True)
            h2d_done[b].record(cp)

    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    cp.wait_event(f0)
    h2d(0)
    for i in range(steps):
        b = i % 2
        stream.wait_event(h2d_done[b])
        if i >= 2:
            stream.wait_event(d2h_done[b])      # od[b] drained by the copy of step i-2
        step(0, x=xd[b], p=pd[b], o=od[b])
        comp_done[b].record(stream)
        if i + 1 < steps:
            if i >= 1:
                cp.wait_event(comp_done[(i + 1) % 2])   # step i-1 has read xd[(i+1) % 2]
            h2d(i + 1)
        with torch.cuda.stream(cp):
            cp.wait_event(comp_done[b])
            oh[b].copy_(od[b], non_blocking=True)
            d2h_done[b].record(cp)
    stream.wait_stream(cp)
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return f0.elapsed_time(f1)


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    import bit_compressed_decode_b200 as fg
    import seeded_inputs as si
    from bit_compressed_decode_b200 import replicas

    rank, world, local = replicas.env_ranks()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", timeout_s=300, device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    h, H, F, P = wl["hidden"], wl["heads"], wl["ffn"], wl["prompt"]
    nb, gbs = wl["nb"], wl["gbs"]
    S = nb * gbs                      # sequences of this rank: its block
    seq0, _ = replicas.shard(world * S, world, rank)
    d = h // H
    nsteps_cfg = wl["steps"]
    maxL = (P + nsteps_cfg + 63) // 64 * 64
    G = args.group
    act_bits = wl.get("act_bits", 16)
    cfg = fg.LayerConfig(h, H, F, group=G, act_bits=act_bits)

    # weights: the shared seeded host generator (same on every rank: replicas)
    w16 = si.layer_weights_f16(0, h, F)
    lw = fg.LayerWeights.from_fp16(cfg, w16, device=dev)
    del w16
    cache = fg.KVCache(S, H, d, maxL, device=dev, group=G)
    # prompt hidden states: seeded device generator (bulk synthetic N(0,1)), per rank
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + seq0)
    zero = torch.zeros(S, dtype=torch.int32, device=dev)
    chunk = max(1, 65536 // P)
    pws = torch.empty(cfg.workspace_bytes(chunk * P), dtype=torch.uint8, device=dev)
    for s0 in range(0, S, chunk):
        n = min(chunk, S - s0)
        xp = torch.randn((n, P, h), generator=g, device=dev, dtype=torch.float16)
        fg.fg_layer_prefill(cfg, lw, cache.view(s0, n), xp, zero[:n], workspace=pws)
        del xp
    del pws
    fg.fg_sync_status()

    xs = [torch.randn((S, h), generator=g, device=dev, dtype=torch.float16) for _ in range(4)]
    pos = [torch.full((S,), P + t, dtype=torch.int32, device=dev) for t in range(nsteps_cfg)]
    out = torch.empty((S, h), dtype=torch.float16, device=dev)
    ws = torch.empty(cfg.workspace_bytes(S), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, x=None, o=None, p=None):
        fg.fg_layer_decode(cfg, lw, cache, xs[i % 4] if x is None else x, pos[i % nsteps_cfg] if p is None else p,
                           num_gpu_batches=nb, gpu_batch_size=gbs, out=out if o is None else o, workspace=ws,
                           stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    fg.fg_sync_status()

    # ---- timed region (device time, CUDA events on the launching stream) ----
    # The steps are timed without per-kernel events; a second timed pass over the same steps
    # with the library's per-kernel events (on the launching stream) gives the breakdown
    # behind the roofline figures.
    sampler = ClockSampler(dev.index if world == 1 else local)
    sampler.start()
    time.sleep(0.3)

    def timed(profile):
        fg.fg_profile_enable(profile)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        fg.fg_profile_enable(False)
        return replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)

    ms = timed(False)
    ms_profiled = timed(True)
    clocks = sampler.stop()
    prof = fg.fg_profile_collect()
    fg.fg_sync_status()
    ms_per_step = ms / args.steps
    value = world * S * args.steps / (ms / 1e3)

    # ---- end to end through host buffers: every step's inputs H2D from pinned memory and its
    # output D2H, on a copy stream with two device input and output buffers, so the copies of
    # steps i+1 and i-1 overlap the decode of step i (events order the two streams) ----
    e2e = run_e2e(torch, fg, step, stream, dev, xs, S, h, P, nsteps_cfg, args.steps, args.warmup, barrier)
    ems = replicas.max_over_ranks(e2e, device=dev)
    e2e_value = world * S * args.steps / (ems / 1e3)
    h2d = S * h * 2 + S * 4
    d2h = S * h * 2

    # ---- roofline of the dominant kernel (and of every kernel) ----
    peaks = load_peaks()
    L_avg = P + (args.warmup + (args.steps - 1) / 2.0) % nsteps_cfg + 1
    # the layer appends decode rows inside the attention kernel only when its (row, head) CTAs
    # are at most 4 per SM (launch-bound); larger blocks take the separate append kernel
    fused = S * wl["heads"] <= 4 * torch.cuda.get_device_properties(dev).multi_processor_count
    work, totals = kernel_work(wl, S, L_avg, G, fused_append=fused)
    kernels = {}
    for name, (tot_ms, cnt) in prof.items():
        if cnt == 0:
            continue
        avg_s = tot_ms / cnt / 1e3
        bound, units = work[name]
        if bound == "tensor":
            # the timed region is ~10 ms at full clock: the burst GEMM peak applies
            ach, peak, unit = units / avg_s / 1e12, peaks["tc_burst"], "TFLOP/s"
        elif bound == "tensor_i8":
            # int8 products: the measured fp16 peak x 2, the nominal int8 / fp16 dense ratio
            ach, peak, unit = units / avg_s / 1e12, peaks["tc_burst"] * 2, "TOP/s"
        else:
            ach, peak, unit = units / avg_s / 1e9, peaks["hbm"], "GB/s"
        kernels[name] = {"bound": bound, "avg_us": round(avg_s * 1e6, 2), "launches": cnt,
                         "share": round(tot_ms / max(1e-9, sum(v[0] for v in prof.values())), 4),
                         "achieved": round(ach, 1), "peak": peak, "unit": unit, "frac": round(ach / peak, 4)}
        if bound == "tensor":
            kernels[name]["frac_of_sustained"] = round(ach / peaks["tc_sustained"], 4)
        elif bound == "tensor_i8":
            kernels[name]["frac_of_sustained"] = round(ach / (2 * peaks["tc_sustained"]), 4)
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    kd = kernels[dom]
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"], "peak": kd["peak"],
                "unit": kd["unit"], "frac": kd["frac"],
                "traffic": read_traffic(dom, args.workload, kernel_units(wl, S, L_avg)[dom]),
                "peak_source": f"{peaks['source']} ({'burst bf16 GEMM' if kd['bound'] == 'tensor' else 'copy'})"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # one sampled sequence per host thread (the oracle splits a step's rows by sequence)
        threads = os.cpu_count() or 1
        n = max(1, min(threads, 32, S))
        osample = OracleSample(wl, n, n)
        t = min(osample.step() for _ in range(2))
        one = OracleSample(wl, 1, 1)
        t1 = one.step()
        cpu = {"value": n / t, "unit": "tokens/s", "cores": n, "kind": "oracle",
               "sample": f"{n} of {S} sequences, one decode step at position {P} ({n} threads, one per sequence)",
               "single_thread": {"value": 1.0 / t1, "unit": "tokens/s", "cores": 1,
                                 "sample": f"1 of {S} sequences, one decode step at position {P}, one thread"}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8 products, f16 elsewhere" if act_bits == 8 else "f16",
            "data": "synthetic",
            "config": {"workload": args.workload, "block": f"{nb}x{gbs}", "sequences_per_gpu": S, "hidden": h,
                       "heads": H, "ffn": F, "prompt": P, "positions": f"{P}..{P + nsteps_cfg - 1} (cycled)",
                       "weights": f"W4 g{G}" + (" (W4A8 form)" if act_bits == 8 else ""),
                       "activations": "int8, one scale per row" if act_bits == 8 else "fp16",
                       "kv": f"KV4 g{G}", "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (KV4 cache %.2f GB + W4 %.0f MB per step)" % (
                           cache.nbytes() / 1e9, totals["w4_bytes"] / 1e6)},
            "roofline": roofline,
            "kernels": kernels,
            "kernels_pass_ms_per_step": ms_profiled / args.steps,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": sum(v[1] for v in prof.values()),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_prefill(args, wl):
    """One step = the prefill of the whole block's prompts through one layer (fg_layer_prefill:
    the same kernels as decode with every prompt row a query, K/V of the prompt appended as 4-bit
    codes), timed with CUDA events; then a second pass with per-kernel events."""
    import torch

    import bit_compressed_decode_b200 as fg
    import seeded_inputs as si
    from bit_compressed_decode_b200 import replicas

    rank, world, local = replicas.env_ranks()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", timeout_s=300, device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    h, H, F, P = wl["hidden"], wl["heads"], wl["ffn"], wl["prompt"]
    nb, gbs = wl["nb"], wl["gbs"]
    S, d = nb * gbs, h // H
    maxL = (P + wl["steps"] + 63) // 64 * 64
    act_bits = wl.get("act_bits", 16)
    cfg = fg.LayerConfig(h, H, F, act_bits=act_bits)
    w16 = si.layer_weights_f16(0, h, F)
    lw = fg.LayerWeights.from_fp16(cfg, w16, device=dev)
    del w16
    cache = fg.KVCache(S, H, d, maxL, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(3000 + rank)
    x = torch.randn((S, P, h), generator=g, device=dev, dtype=torch.float16)
    out = torch.empty_like(x)
    zero = torch.zeros(S, dtype=torch.int32, device=dev)
    # scratch for 64 Ki prompt rows; the library runs the block in chunks of whole sequences
    ws = torch.empty(cfg.workspace_bytes(65536), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        fg.fg_layer_prefill(cfg, lw, cache, x, zero, num_gpu_batches=nb, gpu_batch_size=gbs, out=out, workspace=ws,
                            stream=stream)

    for _ in range(args.warmup):
        step()
    fg.fg_sync_status()
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)

    def timed(profile):
        fg.fg_profile_enable(profile)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        fg.fg_profile_enable(False)
        return replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)

    ms = timed(False)
    ms_profiled = timed(True)
    clocks = sampler.stop()
    prof = fg.fg_profile_collect()
    fg.fg_sync_status()
    peaks = load_peaks()
    rows = S * P
    work, _ = kernel_work(wl, rows, (P + 1) / 2, fused_append=False)   # causal: row t of a prompt reads t + 1 cached tokens
    # prompt attention runs tiled on the tensor cores: 4 d flops per (row, head, visible key)
    # (q.k and p.v), causal, so sum over rows of t + 1 keys; bound by the tensor pipe
    work["attention"] = ("tensor", 4 * (h // H) * H * S * P * (P + 1) // 2)
    kernels = {}
    for name, (tot_ms, n) in prof.items():
        if n == 0:
            continue
        bound, w = work[name]
        per_step_s = tot_ms / 1e3 / args.steps
        if bound == "tensor":
            ach, unit, peak = w / per_step_s / 1e12, "TFLOP/s", peaks["tc_burst"]
        elif bound == "tensor_i8":
            ach, unit, peak = w / per_step_s / 1e12, "TOP/s", peaks["tc_burst"] * 2
        else:
            ach, unit, peak = w / per_step_s / 1e9, "GB/s", peaks["hbm"]
        kernels[name] = {"bound": bound, "ms_per_step": round(tot_ms / args.steps, 3), "launches": n,
                         "share": round(tot_ms / sum(v[0] for v in prof.values()), 4), "achieved": round(ach, 1),
                         "peak": peak, "unit": unit, "frac": round(ach / peak, 4)}
        if bound == "tensor":
            kernels[name]["frac_of_sustained"] = round(ach / peaks["tc_sustained"], 4)
    top = max(kernels, key=lambda n: kernels[n]["share"])
    if rank == 0:
        print(json.dumps({
            "metric": "prefill prompt tokens/s per OPT layer block (W4 KV4)",
            "value": world * rows * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8 products, f16 elsewhere" if act_bits == 8 else "f16",
            "data": "synthetic",
            "config": {"workload": args.workload, "block": f"{nb}x{gbs}", "prompt": P, "hidden": h, "heads": H,
                       "ffn": F, "weights": "W4 g64" + (" (W4A8 form)" if act_bits == 8 else ""),
                       "activations": "int8, one scale per row" if act_bits == 8 else "fp16",
                       "kv": "KV4 g64 written from position 0",
                       "l2": "inputs larger than L2 (prompt activations 2.1 GB per step)"},
            "roofline": {"kernel": top, "bound": kernels[top]["bound"], "achieved": kernels[top]["achieved"],
                         "peak": kernels[top]["peak"], "unit": kernels[top]["unit"], "frac": kernels[top]["frac"],
                         "traffic": None},
            "kernels": kernels, "kernels_pass_ms_per_step": ms_profiled / args.steps,
            "gpu_launches": sum(v[1] for v in prof.values()), "clocks": clocks,
        }), flush=True)


def run_stack(args, wl):
    """One decode step = all layers of the stack for every sequence of the block, each layer's
    packed weights copied from pinned host memory (fg_stack_decode, double-buffered prefetch)."""
    import torch

    import bit_compressed_decode_b200 as fg
    from bit_compressed_decode_b200 import replicas

    rank, world, local = replicas.env_ranks()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", timeout_s=600, device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    h, H, F, P, nl = wl["hidden"], wl["heads"], wl["ffn"], wl["prompt"], args.layers or wl["layers"]
    nb, gbs = wl["nb"], wl["gbs"]
    S, d = nb * gbs, h // H
    maxL = (P + wl["steps"] + 63) // 64 * 64
    act_bits = wl.get("act_bits", 16)
    cfg = fg.LayerConfig(h, H, F, act_bits=act_bits)
    ng = d // 64
    kv_host = bool(wl.get("kv_host"))
    if kv_host and not args.layers:
        # as many layers as half the host's available memory holds (pinned buffers are
        # rounded up to powers of two by torch's host allocator)
        def p2(n):
            return 1 << (int(n) - 1).bit_length()
        per_layer = p2(cfg.blob_bytes()) + 2 * p2(S * H * maxL * d // 2) + 4 * p2(S * H * maxL * ng * 2)
        with open("/proc/meminfo") as f:
            avail = next(int(ln.split()[1]) * 1024 for ln in f if ln.startswith("MemAvailable"))
        nl = max(2, min(nl, int(avail * 0.5) // per_layer))
    # --resident-layers: that many layers (or, with "auto", as many as the device memory left
    # after the KV caches, the staging blobs and caches and 4 GiB of scratch holds) keep their
    # blobs in HBM, spread evenly over the stack
    from bit_compressed_decode_b200 import placement
    if args.resident_layers == "auto":
        kv_layer = S * H * maxL * 2 * (d // 2 + 4 * ng)
        reserve = (2 * kv_layer if kv_host else nl * kv_layer) + 2 * cfg.blob_bytes() + (4 << 30)
        nres = placement.resident_count(torch.cuda.mem_get_info(dev)[0], cfg.blob_bytes(), nl,
                                         reserve_bytes=reserve)
    else:
        nres = min(int(args.resident_layers), nl)
    resident = placement.spread(nres, nl)
    g = torch.Generator(device=dev)
    g.manual_seed(2000 + rank)
    # weights: seeded device draws N(0, 0.02) (biases 0, LayerNorm 1/0), quantised by fg_quantize,
    # then parked in pinned host memory -- the stack streams them back every step
    host = []
    tmp = fg.LayerWeights(cfg, torch.empty(cfg.blob_bytes(), dtype=torch.uint8, device=dev))
    for _ in range(nl):
        for name, shape in (("wqkv", (3 * h, h)), ("wo", (h, h)), ("w1", (F, h)), ("w2", (h, F))):
            w = torch.randn(shape, generator=g, device=dev, dtype=torch.float16) * 0.02
            if act_bits == 8:
                fg.fg_w4a8_quantize_weight(w, out=tmp.w4a8_matrix(name))
            else:
                fg.fg_quantize(w, dim=1, out=tmp.matrix(name))
            del w
        for name in ("bqkv", "bo", "b1", "b2", "ln1_b", "ln2_b"):
            tmp.vector(name).zero_()
        tmp.vector("ln1_g").fill_(1.0)
        tmp.vector("ln2_g").fill_(1.0)
        # a resident layer keeps its blob in device memory (read in place); spread evenly, the
        # copy of a streamed layer overlaps the compute of the resident one before it
        if resident[len(host)]:
            hb = tmp.blob.clone()
        else:
            hb = torch.empty(cfg.blob_bytes(), dtype=torch.uint8, pin_memory=True)
            hb.copy_(tmp.blob)
        host.append(hb)
    del tmp
    torch.cuda.synchronize()
    nbuf = 2 if kv_host else args.staging_buffers   # the host-KV stack alternates two staging caches
    st = fg.Stack(cfg, host, device=dev, staging_buffers=nbuf)
    # KV caches: seeded random codes and group min/scale for the prompt positions (a decode
    # step reads the same bytes whatever they hold; prefilling 48 layers x 512 tokens through
    # the per-row attention kernel would take far longer than the timed steps)

    def seeded_cache():
        return fg.KVCache(S, H, d, maxL, device=dev, arrays=[
            torch.randint(0, 256, (S, H, maxL, d // 2), generator=g, device=dev, dtype=torch.uint8),
            torch.randn((S, H, maxL, ng), generator=g, device=dev, dtype=torch.float16),
            (torch.rand((S, H, maxL, ng), generator=g, device=dev) * 0.2).half(),
            torch.randint(0, 256, (S, H, maxL, d // 2), generator=g, device=dev, dtype=torch.uint8),
            torch.randn((S, H, maxL, ng), generator=g, device=dev, dtype=torch.float16),
            (torch.rand((S, H, maxL, ng), generator=g, device=dev) * 0.2).half()])

    caches, staging = [], []
    if kv_host:
        # every layer's cache drawn on the device, then parked in its own pinned host arrays
        for _ in range(nl):
            c = seeded_cache()
            hc = fg.KVCache(S, H, d, maxL, device="cpu", pin_memory=True)
            for a, b in zip(hc.arrays(), c.arrays()):
                a.copy_(b)
            caches.append(hc)
            del c
        staging = [fg.KVCache(S, H, d, maxL, device=dev) for _ in range(2)]
    else:
        caches = [seeded_cache() for _ in range(nl)]
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=dev)
    fg.fg_sync_status()
    xs = [torch.randn((S, h), generator=g, device=dev, dtype=torch.float16) for _ in range(2)]
    pos = [torch.full((S,), P + t, dtype=torch.int32, device=dev) for t in range(wl["steps"])]
    out = torch.empty((S, h), dtype=torch.float16, device=dev)
    ws = torch.empty(st.workspace_bytes(S), dtype=torch.uint8, device=dev)

    def step(i):
        t = i % wl["steps"]
        if kv_host:
            # positions [0, P+t) filled before each layer, slot P+t written back after it
            st.decode_host_kv(caches, staging, xs[i % 2], pos[t], P + t, P + t, P + t + 1, num_gpu_batches=nb,
                              gpu_batch_size=gbs, out=out, workspace=ws, compute_stream=compute, copy_stream=copy)
        else:
            st.decode(caches, xs[i % 2], pos[t], num_gpu_batches=nb, gpu_batch_size=gbs, out=out,
                      workspace=ws, compute_stream=compute, copy_stream=copy)

    # host-link peak: a plain pinned -> device cudaMemcpyAsync of 1 GiB on the copy stream
    # (best of 5), the denominator of the stack's roofline
    pin = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    link = []
    for _ in range(5):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(copy)
        with torch.cuda.stream(copy):
            dst.copy_(pin, non_blocking=True)
        c1.record(copy)
        c1.synchronize()
        link.append(c0.elapsed_time(c1))
    link_peak = (1 << 30) / (min(link) / 1e3) / 1e9
    del pin, dst

    for i in range(args.warmup):
        step(i)
    fg.fg_sync_status()
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    for i in range(args.steps):
        step(args.warmup + i)
    e1.record(compute)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)
    fg.fg_sync_status()
    blob_gb = cfg.blob_bytes() * (nl - nres) / 1e9
    slot_bytes = S * H * 2 * (d // 2 + 4 * ng)          # K and V codes + min/scale of one position
    fill_gb = wb_gb = 0.0
    if kv_host:
        ts = [(args.warmup + i) % wl["steps"] for i in range(args.steps)]
        fill_gb = sum((P + t) * slot_bytes for t in ts) * nl / args.steps / 1e9
        wb_gb = slot_bytes * nl / 1e9
    if rank == 0:
        line = {
            "metric": ("decode tokens/s of the OPT layer stack (W4 weights and KV4 streamed from pinned host)"
                       if kv_host else
                       "decode tokens/s of the OPT layer stack (W4 weights streamed from pinned host, KV4 in HBM)"),
            "value": world * S * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "dtype": "i8 products, f16 elsewhere" if act_bits == 8 else "f16", "data": "synthetic",
            "config": {"workload": args.workload, "layers": nl, "block": f"{nb}x{gbs}", "hidden": h, "prompt": P,
                       "weights_streamed_gb_per_step": round(blob_gb, 3),
                       "staging_buffers": f"{nbuf} x {st.staging[0].numel() / 1e9:.3f} GB",
                       "resident_layers": nres,
                       "kv": "KV4 g64, seeded random codes at the prompt positions (no prefill)"},
            "host_link_gbs": round((blob_gb + fill_gb + wb_gb) / (ms / args.steps / 1e3), 1),
            "roofline": ({"bound": "host-link", "achieved": round((blob_gb + fill_gb) / (ms / args.steps / 1e3), 1),
                          "peak": round(link_peak, 1), "unit": "GB/s",
                          "frac": round((blob_gb + fill_gb) / (ms / args.steps / 1e3) / link_peak, 4),
                          "traffic": None,
                          "peak_source": "measured here: pinned host -> device cudaMemcpyAsync of 1 GiB"}
                         if blob_gb + fill_gb > 0 else
                         {"bound": None, "note": "every layer resident in HBM: nothing crosses the host link; "
                                                 "the layer kernels' own rooflines apply (see the decode workloads)"}),
            "clocks": clocks,
        }
        if kv_host:
            line["config"]["kv_fill_gb_per_step"] = round(fill_gb, 3)
            line["config"]["kv_writeback_gb_per_step"] = round(wb_gb, 4)
            line["config"]["kv_gb_in_host"] = round(sum(c.nbytes() for c in caches) / 1e9, 2)
            # the same per-layer time over the model's full depth (every layer moves the same bytes)
            line["tokens_per_s_full_depth_projected"] = line["value"] * nl / wl["model_layers"]
            line["config"]["model_layers"] = wl["model_layers"]
        else:
            line["config"]["kv_gb_in_hbm"] = round(sum(c.nbytes() for c in caches) / 1e9, 2)
        print(json.dumps(line), flush=True)
    st.close()


def run_kernel(args, wl):
    """Standalone launches of one kernel of the decode step on the workload's shapes,
    timed with CUDA events (used for per-kernel measurements and small ncu captures)."""
    import torch

    import bit_compressed_decode_b200 as fg
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    h, H, F, P = wl["hidden"], wl["heads"], wl["ffn"], wl["prompt"]
    S = args.seqs or wl["nb"] * wl["gbs"]
    d = h // H
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    if args.kernel in ("attention", "attention_append"):
        maxL = (P + wl["steps"] + 63) // 64 * 64
        ng = d // 64
        cache = fg.KVCache(S, H, d, maxL, device=dev, arrays=[
            torch.randint(0, 256, (S, H, maxL, d // 2), generator=g, device=dev, dtype=torch.uint8),
            torch.randn((S, H, maxL, ng), generator=g, device=dev, dtype=torch.float16),
            (torch.rand((S, H, maxL, ng), generator=g, device=dev) * 0.2).half(),
            torch.randint(0, 256, (S, H, maxL, d // 2), generator=g, device=dev, dtype=torch.uint8),
            torch.randn((S, H, maxL, ng), generator=g, device=dev, dtype=torch.float16),
            (torch.rand((S, H, maxL, ng), generator=g, device=dev) * 0.2).half()])
        qkv = torch.randn((S, 3 * h), generator=g, device=dev, dtype=torch.float16) * 0.1
        out = torch.empty((S, h), dtype=torch.float16, device=dev)
        pos = torch.full((S,), P, dtype=torch.int32, device=dev)
        kv_tok = 2 * (d // 2 + 4 * ng)
        work, unit, peak = S * H * (P + 1) * kv_tok + 2 * S * h * 2, "GB/s", peaks["hbm"]
        if args.kernel == "attention":
            run = lambda: fg.fg_attention_decode(cache, qkv[:, :h], pos, out=out, stream=stream)
        else:  # the decode step's form: the new k, v appended at position P in the same launch
            run = lambda: fg.fg_attention_decode_append(cache, qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:], pos,
                                                        out=out, stream=stream)
            work += 2 * S * h * 2 + S * H * kv_tok
    elif args.kernel == "prefill_attention":
        # the prompts' attention of the prefill: S sequences x P prompt rows over a cache holding
        # those P tokens (seeded codes), causal; 4 d flops per (row, head, visible key)
        maxL = (P + 63) // 64 * 64
        ng = d // 64
        cache = fg.KVCache(S, H, d, maxL, device=dev, arrays=[
            torch.randint(0, 256, (S, H, maxL, d // 2), generator=g, device=dev, dtype=torch.uint8),
            torch.randn((S, H, maxL, ng), generator=g, device=dev, dtype=torch.float16),
            (torch.rand((S, H, maxL, ng), generator=g, device=dev) * 0.2).half(),
            torch.randint(0, 256, (S, H, maxL, d // 2), generator=g, device=dev, dtype=torch.uint8),
            torch.randn((S, H, maxL, ng), generator=g, device=dev, dtype=torch.float16),
            (torch.rand((S, H, maxL, ng), generator=g, device=dev) * 0.2).half()])
        q = torch.randn((S * P, h), generator=g, device=dev, dtype=torch.float16) * 0.1
        out = torch.empty((S * P, h), dtype=torch.float16, device=dev)
        zero = torch.zeros((S,), dtype=torch.int32, device=dev)
        run = lambda: fg.fg_attention_decode(cache, q, zero, rows_per_seq=P, out=out, stream=stream)
        work, unit, peak = 4 * d * H * S * P * (P + 1) // 2, "TFLOP/s", peaks["tc_burst"]
    elif args.kernel.endswith("_gemm_w4a8"):
        # the W4A8 variant of a decode GEMM: int8 activations (quantised once, outside the timed
        # launches) times two-level 4-bit weights on the integer tensor cores; the peak is the
        # measured fp16 GEMM peak x 2, the nominal int8 / fp16 dense ratio (4.5 / 2.25 PFLOP/s)
        N, K = {"qkv": (3 * h, h), "out": (h, h), "fc1": (F, h), "fc2": (h, F)}[args.kernel[:-len("_gemm_w4a8")]]
        x = torch.randn((S, K), generator=g, device=dev, dtype=torch.float16)
        wq = fg.fg_w4a8_quantize_weight(torch.randn((N, K), generator=g, device=dev, dtype=torch.float16) * 0.02)
        a8, asc = fg.fg_act8_quantize(x)
        y = torch.empty((S, N), dtype=torch.float16, device=dev)
        run = lambda: fg.fg_linear_w4a8(a8, asc, wq, out=y, stream=stream)
        work, unit, peak = 2 * S * N * K, "TOP/s", peaks["tc_burst"] * 2
    elif args.kernel == "act8_quantize":
        x = torch.randn((S, F), generator=g, device=dev, dtype=torch.float16)
        a8, asc = fg.fg_act8_quantize(x)
        run = lambda: fg.fg_act8_quantize(x, a8, asc, stream=stream)
        work, unit, peak = S * F * 3 + S * 4, "GB/s", peaks["hbm"]
    elif args.kernel.endswith("_gemm"):
        N, K = {"qkv_gemm": (3 * h, h), "out_gemm": (h, h), "fc1_gemm": (F, h), "fc2_gemm": (h, F)}[args.kernel]
        x = torch.randn((S, K), generator=g, device=dev, dtype=torch.float16)
        wq = fg.fg_quantize(torch.randn((N, K), generator=g, device=dev, dtype=torch.float16) * 0.02, dim=1,
                            group=args.group)
        y = torch.empty((S, N), dtype=torch.float16, device=dev)
        # --gemm-scratch: auto = the full scratch; persistent = the full scratch and the persistent
        # launch; classic = the classic launch's split-k scratch only; none = splits added on chip
        M_, N_, K_ = x.shape[0], wq.shape[0], x.shape[1]
        nbytes = {"auto": fg.fg_linear_workspace_bytes(M_, N_, K_), "persistent": fg.fg_linear_workspace_bytes(M_, N_, K_),
                  "classic": fg.fg_linear_classic_scratch_bytes(M_, N_, K_), "none": 0}[args.gemm_scratch]
        gws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=dev)
        persistent = args.gemm_scratch == "persistent"
        run = lambda: fg.fg_linear_w4a16(x, wq, out=y, workspace=gws, stream=stream, persistent=persistent)
        work, unit, peak = 2 * S * N * K, "TFLOP/s", peaks["tc_burst"]
    elif args.kernel in ("quantize", "dequantize"):
        n = 1 << args.log2_elems
        x = torch.randn((n // 4096, 4096), generator=g, device=dev, dtype=torch.float16) * 0.02
        q = fg.fg_quantize(x, group=args.group, bits=args.bits)
        if args.kernel == "quantize":
            run = lambda: fg.fg_quantize(x, group=args.group, bits=args.bits, out=q, stream=stream)
        else:
            run = lambda: fg.fg_dequantize(q, stream=stream)
        work, unit, peak = n * (2 + args.bits / 8 + 4.0 / args.group), "GB/s", peaks["hbm"]
    else:
        raise SystemExit(f"unknown kernel {args.kernel}")
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        run()
        b.record(stream)
    torch.cuda.synchronize()
    fg.fg_sync_status()
    t = sorted(a.elapsed_time(b) / 1e3 for a, b in ev)
    med = t[len(t) // 2]
    scale = 1e12 if unit in ("TFLOP/s", "TOP/s") else 1e9
    line = {"kernel": args.kernel, "group": args.group, "workload": args.workload, "seqs": S,
            "gemm_scratch": args.gemm_scratch if args.kernel.endswith("_gemm") else None,
            "plan": fg.fg_linear_w4a8_plan(S, N, K) if args.kernel.endswith("_gemm_w4a8") else None,
            "median_us": med * 1e6,
            "min_us": t[0] * 1e6, "achieved": work / med / scale, "unit": unit, "peak": peak,
            "frac": work / med / scale / peak}
    if args.kernel in ("quantize", "dequantize") and not args.no_cpu_baseline:
        line["log2_elems"] = args.log2_elems
        line["bits"] = args.bits
        line["cpu_baseline"] = oracle_quant_baseline(args.kernel, args.group, args.log2_elems, args.bits)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="opt-6.7b-layer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", default=None,
                    help="time one kernel alone: attention, attention_append, prefill_attention, qkv_gemm, out_gemm, fc1_gemm, "
                         "fc2_gemm, quantize, dequantize")
    ap.add_argument("--seqs", type=int, default=0, help="--kernel: sequences (default: the workload's block)")
    ap.add_argument("--log2-elems", type=int, default=28, help="--kernel quantize/dequantize: tensor size")
    ap.add_argument("--bits", type=int, choices=(4, 8), default=4, help="--kernel quantize/dequantize: code width")
    ap.add_argument("--layers", type=int, default=0, help="stack workloads: number of layers (default: the model's)")
    ap.add_argument("--group", type=int, choices=(64, 128), default=64,
                    help="quantisation group size: of the layer's weights and KV cache (layer workloads), or of "
                         "--kernel quantize/dequantize/*_gemm")
    ap.add_argument("--resident-layers", default="0",
                    help="stack workloads: layers whose weight blobs stay in device memory (read in place), "
                         "or 'auto': as many as the device memory left holds")
    ap.add_argument("--staging-buffers", type=int, choices=(1, 2), default=2,
                    help="opt-30b-stack: device staging blobs (2 alternate; 1 is refilled slice by slice)")
    ap.add_argument("--gemm-scratch", choices=("auto", "persistent", "classic", "none"), default="auto",
                    help="--kernel *_gemm: the full scratch (auto), the full scratch and the persistent launch "
                         "(persistent), the classic launch's split-k scratch (classic), or none (splits added on chip)")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    if args.kernel:
        run_kernel(args, wl)
    elif wl.get("phase") == "prefill" and args.impl == "ours":
        run_prefill(args, wl)
    elif "layers" in wl and args.impl == "ours":
        run_stack(args, wl)
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
