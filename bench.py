#!/usr/bin/env python
"""Benchmark: routed MoE layer with a GPU (layer, expert) LRU slot cache on B200.

Workload (one step = one moe_layer_forward over one batch: router -> cache
lookup + miss fills from pinned host RAM -> permute -> grouped SwiGLU FFN
over hits, then misses -> combine): the DeepSeek-V4-Flash-shaped MXFP4
decode layer (256 experts, top-6, hidden 4096, FFN 2048), 64 expert slots,
Zipf(1.1) routing through the router bias, batch of 16 tokens, a continuous
decode stream from a cold cache (warm-up steps included).  L2 is flushed
(256 MiB write) before every step, outside the step's events.

Prints one JSON line (rank 0).  --impl reference times the CPU oracle on
one-token samples of the same workload instead.

Multi-GPU: `--gpus N` under torchrun runs N independent replicas (the layer
does not shard: every step of it is local to one GPU); the only collectives
are the timing barrier and the max-over-ranks reduction.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s (decode & prefill); % of HBM / FP4 tensor roofline"
L2_FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--batch", type=int, default=16)
    p.add_argument("--no-extras", action="store_true", help="skip the resident / prefill / batch-sweep legs")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--resident-batch", default="1,4,16", help="batch sizes of the resident decode leg")
    p.add_argument("--leg", choices=["all", "resident", "prefill"], default="all",
                   help="resident / prefill: run only that context leg (profiling); prints its own JSON line")
    return p.parse_args()


def workload_config(cfg, n, world):
    return {"workload": "DeepSeek-V4-Flash-shaped MXFP4 MoE decode layer: 256 routed experts, top-6, "
                        "hidden 4096, expert FFN 2048, 64-slot GPU expert cache (LRU, misses filled from "
                        "pinned host RAM), Zipf(1.1) routing, continuous decode stream from a cold cache",
            "batch_tokens": n, "experts": cfg.experts, "top_k": cfg.top_k, "hidden": cfg.hidden,
            "ffn": cfg.ffn, "weights": "mxfp4", "activations": "bf16", "capacity_slots": cfg.capacity,
            "routing": "zipf(s=1.1) via router bias, seed 0", "l2": "flushed before every step (256 MiB write)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# ------------------------------------------------------------------ clocks
class Clocks:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + ",".join(self.FIELDS),
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t0 = time.time()   # the sampler is running once it has written a line
        while time.time() - t0 < 5 and os.path.getsize(self.path) == 0 and self.proc.poll() is None:
            time.sleep(0.01)

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "samples": len(sm),
                "reasons": sorted(reasons)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor peak (burst) and its provenance; the FFN's f16 MMAs run at the same rate."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ------------------------------------------------------------------ multi-rank plumbing
def max_over_ranks(ms: float, device=None) -> float:
    """The largest per-rank device time (a no-op on one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world: int, steps: int, tokens_per_step: int, ms_max: float) -> float:
    """Whole-job tokens/s: every replica's tokens over the slowest replica's time."""
    return world * steps * tokens_per_step / (ms_max / 1000.0)


# ------------------------------------------------------------------ setup
def build_layer(cfg, seed):
    """Pinned host blobs of every expert, router matrix and bias (seed-fixed weights)."""
    import torch

    from expert_cached_sparse_b200 import api as A
    from expert_cached_sparse_b200 import workloads as W
    shape = A.shape_of(cfg)
    sb = A.moe_slot_bytes(shape)
    blobs = []
    for e in range(cfg.experts):
        b = torch.empty(sb, dtype=torch.uint8, pin_memory=True)
        A.moe_pack_expert(shape, W.gen_expert(cfg, seed, 0, e), out=b.numpy())
        blobs.append(b)
    return shape, blobs, W.gen_wg(cfg, seed, 0), W.gen_bias(cfg, seed, 0)


def to_dev_bits(a, device):
    import torch
    return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)


class DecodeStream:
    """One replica: a cache over the host blobs, device inputs for every step, workspace."""

    def __init__(self, cfg, shape, blobs, wg, bias, n, steps, capacity, rank, device, tag="decode"):
        import torch

        from expert_cached_sparse_b200 import api as A
        from expert_cached_sparse_b200 import workloads as W
        self.A, self.n, self.cfg, self.shape = A, n, cfg, shape
        self.cache = A.MoeCache(shape, capacity, blobs, trace_capacity=0)
        self.wg = to_dev_bits(wg, device)
        self.bias = torch.from_numpy(bias).to(device) if bias is not None else None
        xs = np.stack([W.gen_x(cfg, 1000 + rank, n, tag, s) for s in range(steps)])
        self.x_host = xs
        self.x = to_dev_bits(xs, device)                      # [steps, n, H]
        self.out = torch.empty(n, cfg.hidden, dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(A.moe_layer_workspace_bytes(shape, n), dtype=torch.uint8, device=device)
        self.idx = torch.empty(steps, n, cfg.top_k, dtype=torch.int32, device=device)
        self.stream = torch.cuda.Stream(device)
        self.copy = torch.cuda.Stream(device)
        torch.cuda.synchronize()

    def step(self, s, x=None, out=None):
        self.A.moe_layer_forward(self.cache, 0, self.x[s] if x is None else x, self.wg, self.bias,
                                 self.out if out is None else out, self.ws, stream=self.stream,
                                 copy_stream=self.copy, topk_idx_out=self.idx[s])


# DRAM bytes (read + write) per grouped-FFN call of the headline decode
# stream, summed over the call's kernels (operand preps and both projections)
# and averaged over the calls of an ncu capture of that workload.  Valid only
# for the FFN code it was measured on (comments aside): other code reports null.
FFN_TRAFFIC = {"source_sha1": None, "bytes_per_call": None}


def ffn_source_sha1():
    """SHA-1 of the FFN source with comments and blank lines removed (the code
    the traffic was measured on; comment edits do not change it)."""
    import hashlib
    import re
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "expert_cached_sparse_b200", "csrc", "ffn_fp4.cu")
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha1(code.encode()).hexdigest()


def ffn_traffic():
    return FFN_TRAFFIC["bytes_per_call"] if ffn_source_sha1() == FFN_TRAFFIC["source_sha1"] else None


def ffn_algorithmic_bytes(idx_steps, cfg, slot_bytes):
    """Per-step bytes the grouped FFN must move: each touched expert's weights once,
    x_perm read, h written and read, y_perm written."""
    total = 0
    for idx in idx_steps:
        U = len(np.unique(idx))
        A_ = idx.size
        total += U * slot_bytes + A_ * cfg.hidden * 2 * 2 + A_ * cfg.ffn * 2 * 2
    return total


def timed_steps(ds, first, k, flush, dist_ok):
    """Runs steps first..first+k-1, each after an L2 flush; returns summed device ms."""
    import torch
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
    for i in range(k):
        with torch.cuda.stream(ds.stream):
            flush.zero_()
            starts[i].record(ds.stream)
        ds.step(first + i)
        with torch.cuda.stream(ds.stream):
            ends[i].record(ds.stream)
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends))


def graph_steps(ds, first, k, flush):
    """A fully resident layer step reads nothing back to the host, so it can be
    captured once in a CUDA graph; replays steps first..first+k-1 (inputs copied
    into the captured input buffer before each, outside the events) and returns
    the summed device ms."""
    import torch
    xin = ds.x[first].clone()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=ds.stream):
        ds.step(first, x=xin)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
    for i in range(k):
        with torch.cuda.stream(ds.stream):
            flush.zero_()
            xin.copy_(ds.x[first + i])
            starts[i].record(ds.stream)
            g.replay()
            ends[i].record(ds.stream)
    torch.cuda.synchronize()
    del g
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends))


# ------------------------------------------------------------------ oracle timing
def oracle_token_steps(cfg, seed, n_steps, batch):
    """The CPU oracle, as it stands, on one-token samples of the decode stream:
    each sample routes one token, updates the oracle LRU, dequantises its
    experts, runs their SwiGLU FFNs and combines.  Returns (seconds, tokens)."""
    from expert_cached_sparse_b200 import workloads as W
    from oracle import oracle as O
    O.build()
    wg = W.gen_wg(cfg, seed, 0)
    bias = W.gen_bias(cfg, seed, 0)
    lru = O.Lru(1, cfg.experts, cfg.capacity)
    xs = [W.gen_x(cfg, 1000, batch, "decode", s)[:1] for s in range(n_steps)]
    experts = {}

    def fn(e):
        if e not in experts:
            experts[e] = W.gen_expert(cfg, seed, 0, e)
        return experts[e]

    for s in range(n_steps):           # weights are inputs: generated before the clock starts
        _, idx, _ = O.router(xs[s], wg, bias, cfg.top_k)
        for e in idx.reshape(-1):
            fn(int(e))
    t0 = time.perf_counter()
    for s in range(n_steps):
        out, idx, w, _ = O.moe_layer(xs[s], wg, bias, cfg.top_k, cfg.wfmt, cfg.hidden, cfg.ffn, fn)
        lru.call(0, idx)
    return time.perf_counter() - t0, n_steps


def run_reference(args, cfg, world):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    total = args.steps + args.warmup
    oracle_token_steps(cfg, 0, min(args.warmup, 2), args.batch)      # warm-up samples
    sec, toks = oracle_token_steps(cfg, 0, args.steps, args.batch)
    value = toks / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sec / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg, args.batch, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{args.steps} one-token samples of the decode stream (route, LRU, "
                                       f"dequantise 6 experts, 6 SwiGLU FFNs, combine), single thread"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, cfg, world, rank, local_rank):
    import torch
    import torch.distributed as dist

    from expert_cached_sparse_b200 import api as A
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist_ok = world > 1

    def barrier():
        if dist_ok:
            dist.barrier(device_ids=[local_rank])

    n, K, Wm = args.batch, args.steps, args.warmup
    shape, blobs, wg, bias = build_layer(cfg, 0)
    slot_bytes = A.moe_slot_bytes(shape)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    hbm_peak, peak_kind = measured_peaks()
    if args.leg != "all":
        res = extras(cfg, shape, blobs, wg, bias, K, Wm, flush, device, hbm_peak, legs=(args.leg,),
                     batches=tuple(int(b) for b in args.resident_batch.split(",")))
        if rank == 0:
            print(json.dumps({"leg": args.leg, "steps": K, "warmup": Wm, "results": res}), flush=True)
        return

    # ---- headline: 64-slot decode stream
    ds = DecodeStream(cfg, shape, blobs, wg, bias, n, 2 * K + Wm, cfg.capacity, rank, device)
    for s in range(Wm):
        ds.step(s)
    torch.cuda.synchronize()
    A.moe_profile_read(reset=True)
    A.moe_profile_enable(True)
    st0 = ds.cache.stats()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = int(vis.split(",")[local_rank]) if vis and vis.split(",")[local_rank].isdigit() else local_rank
    clocks = Clocks(smi_index)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    ms = timed_steps(ds, Wm, K, flush, dist_ok)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    prof = A.moe_profile_read(reset=True)
    A.moe_profile_enable(False)
    st1 = ds.cache.stats()
    ms_max = max_over_ranks(ms, device)
    value = throughput(world, K, n, ms_max)
    idx_steps = ds.idx[Wm:Wm + K].cpu().numpy()
    ffn_bytes = ffn_algorithmic_bytes(idx_steps, cfg, slot_bytes)
    ffn_ms = prof["ffn"]["ms"]
    ffn_calls = max(1, prof["ffn"]["timed"])
    achieved = ffn_bytes / (ffn_ms / 1000.0) / 1e9 if ffn_ms > 0 else 0.0
    kernels = sum(prof[k]["launches"] for k in ("router", "lookup", "permute", "ffn", "combine"))
    lookups = st1["lookups"] - st0["lookups"]
    hits = st1["hits"] - st0["hits"]
    misses = st1["misses"] - st0["misses"]
    fill_ms = prof["fill"]["ms"]
    fill_gbs = (st1["fill_bytes"] - st0["fill_bytes"]) / (fill_ms / 1000.0) / 1e9 if fill_ms > 0 else None

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": workload_config(cfg, n, world)}
    line["roofline"] = {"kernel": "grouped SwiGLU FFN (ffn_fp4_kernel gate-up + down, block-scaled tcgen05)",
                        "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                        "frac": achieved / hbm_peak, "peak_kind": peak_kind, "traffic": ffn_traffic(),
                        "algorithmic_bytes_per_call": ffn_bytes / ffn_calls,
                        "avg_call_ms": ffn_ms / ffn_calls, "calls": ffn_calls}
    line["gpu_launches"] = int(kernels)
    line["cache"] = {"lookups": lookups, "hit_rate": hits / max(1, hits + misses), "misses_per_step": misses / K,
                     "fill_GBps": fill_gbs, "fill_ms_per_step": fill_ms / K,
                     "step_ms_breakdown": {k: prof[k]["ms"] / K for k in prof}}
    line["clocks"] = clk

    # ---- e2e through the public API: pinned host x in, host out, every step
    if not args.no_e2e:
        xh = torch.from_numpy(ds.x_host[Wm + K:Wm + 2 * K].view(np.int16)).pin_memory()
        oh = torch.empty(n, cfg.hidden, dtype=torch.int16).pin_memory()
        xd = torch.empty(n, cfg.hidden, dtype=torch.int16, device=device)
        s_, e_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        s_.record(ds.stream)
        for i in range(K):
            with torch.cuda.stream(ds.stream):
                xd.copy_(xh[i], non_blocking=True)
            ds.step(Wm + K + i, x=xd.view(torch.bfloat16))
            with torch.cuda.stream(ds.stream):
                oh.copy_(ds.out.view(torch.int16), non_blocking=True)
            ds.stream.synchronize()
        e_.record(ds.stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(s_.elapsed_time(e_), device)
        line["e2e"] = {"value": throughput(world, K, n, e2e_ms), "unit": "tokens/s",
                       "h2d_bytes_per_step": n * cfg.hidden * 2, "d2h_bytes_per_step": n * cfg.hidden * 2,
                       "note": "no L2 flush; expert fills (misses) are part of the step, not input bytes"}
    ds.cache.close()
    del ds

    # ---- extra legs (rank 0 only, single-GPU context numbers)
    if not args.no_extras and rank == 0:
        line["extras"] = extras(cfg, shape, blobs, wg, bias, K, Wm, flush, device, hbm_peak)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, toks = oracle_token_steps(cfg, 0, 16, n)
        line["cpu_baseline"] = {"value": toks / sec, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{toks} one-token samples of the same decode stream (route, LRU, "
                                          f"dequantise 6 experts, 6 SwiGLU FFNs, combine), "
                                          f"{sec:.1f} s single-threaded"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def extras(cfg, shape, blobs, wg, bias, K, Wm, flush, device, hbm_peak, legs=("resident", "prefill"),
           batches=(1, 4, 16)):
    """Context legs: the same layer with every expert resident (HBM-bound decode)
    at batch 1, 4 and 16, and the 4096-token prefill."""
    import torch

    from expert_cached_sparse_b200 import api as A
    from expert_cached_sparse_b200 import workloads as W
    out = {}
    slot_bytes = A.moe_slot_bytes(shape)
    # resident decode (256 slots, all experts preloaded)
    for n in (batches if "resident" in legs else ()):
        ds = DecodeStream(cfg, shape, blobs, wg, bias, n, K + Wm, cfg.experts, 0, device, tag="resident")
        ds.cache.lookup_update(0, torch.arange(cfg.experts, dtype=torch.int32, device=device))
        torch.cuda.synchronize()
        for s in range(Wm):
            ds.step(s)
        torch.cuda.synchronize()
        A.moe_profile_read(reset=True)
        A.moe_profile_enable(True)
        ms = timed_steps(ds, Wm, K, flush, False)
        prof = A.moe_profile_read(reset=True)
        A.moe_profile_enable(False)
        idx = ds.idx[Wm:Wm + K].cpu().numpy()
        fb = ffn_algorithmic_bytes(idx, cfg, slot_bytes)
        layer_bytes = fb + K * (cfg.experts * cfg.hidden * 2 + 2 * n * cfg.hidden * 2)
        graph_ms = graph_steps(ds, Wm, K, flush)
        out[f"resident_decode_b{n}"] = {
            "tokens_per_s": K * n / (ms / 1000), "ms_per_step": ms / K,
            "layer_hbm_frac": layer_bytes / (ms / 1000) / 1e9 / hbm_peak,
            "ffn_GBps": fb / (prof["ffn"]["ms"] / 1000) / 1e9, "ffn_hbm_frac": fb / (prof["ffn"]["ms"] / 1000) / 1e9 / hbm_peak,
            "cuda_graph": {"tokens_per_s": K * n / (graph_ms / 1000), "ms_per_step": graph_ms / K,
                           "note": "the same resident steps captured once in a CUDA graph and replayed "
                                   "(one replay per step, L2 flushed before each, profiling off)"},
            "unique_experts_per_step": float(np.mean([len(np.unique(i)) for i in idx])),
            "step_ms_breakdown": {k: prof[k]["ms"] / K for k in prof}}
        ds.cache.close()
        del ds
    if "prefill" not in legs:
        return out
    # prefill: 4096 tokens, Zipf(0.8), all experts resident
    pcfg = W.DS_PREFILL
    pbias = W.gen_bias(pcfg, 0, 0)
    n = 4096
    steps = 3
    ds = DecodeStream(pcfg, shape, blobs, wg, pbias, n, steps + 1, pcfg.experts, 0, device, tag="prefill")
    ds.cache.lookup_update(0, torch.arange(cfg.experts, dtype=torch.int32, device=device))
    ds.step(0)
    torch.cuda.synchronize()
    A.moe_profile_read(reset=True)
    A.moe_profile_enable(True)
    ms = timed_steps(ds, 1, steps, flush, False)
    prof = A.moe_profile_read(reset=True)
    A.moe_profile_enable(False)
    idx = ds.idx[1:1 + steps].cpu().numpy()
    flops = steps * n * cfg.top_k * 3 * 2 * cfg.hidden * cfg.ffn
    tensor_peak, tensor_kind = measured_bf16_tflops()
    out["prefill_4096"] = {"tokens_per_s": steps * n / (ms / 1000), "ms_per_step": ms / steps,
                           "ffn_tflops": flops / (prof["ffn"]["ms"] / 1000) / 1e12,
                           "ffn_tensor_frac": flops / (prof["ffn"]["ms"] / 1000) / 1e12 / tensor_peak,
                           "tensor_peak_tflops": tensor_peak, "tensor_peak_kind": tensor_kind,
                           "unique_experts_per_step": float(np.mean([len(np.unique(i)) for i in idx])),
                           "step_ms_breakdown": {k: prof[k]["ms"] / steps for k in prof}}
    ds.cache.close()
    return out


def main():
    args = parse()
    from expert_cached_sparse_b200 import workloads as W
    cfg = W.DS_DECODE
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        if world == 1 and args.gpus > 1:
            print(json.dumps({"error": "--gpus > 1 must be launched with torchrun"}), flush=True)
            return 2
    if args.impl == "reference":
        return run_reference(args, cfg, world)
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, cfg, world, rank, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
