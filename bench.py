#!/usr/bin/env python
"""Benchmark: routed MoE layer with a GPU (layer, expert) LRU slot cache on B200.

Headline (one step = one moe_layer_forward over one batch: router -> cache
lookup + miss fills from pinned host RAM -> permute -> grouped SwiGLU FFN
over hits, then misses -> combine): the DeepSeek-V4-Flash-shaped MXFP4
decode layer (256 experts, top-6, hidden 4096, FFN 2048), 64 expert slots,
Zipf(1.1) routing through the router bias, batch of 16 tokens, a continuous
decode stream from a cold cache (warm-up steps included).  L2 is flushed
(256 MiB write) before every step, outside the step's events.

Context legs (`extras`, rank 0): every other workload of the layer --
the tiny BF16 layer, the same decode layer fully resident at batch 1/4/16,
its 4096-token prefill, the Qwen-shaped BF16 layer (512-token prefill and
8-token decode), and the 40-layer NVFP4 decode trace with its 1024-slot
cache -- each with its roofline fraction and the CPU oracle's rate on a
bounded sample (pinned to one core).  The pinned host->device bandwidth Bp
is measured in the run.

Prints one JSON line (rank 0).  --impl reference times the CPU oracle on
one-token samples of the headline workload instead.

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
    p.add_argument("--leg", choices=["all", "resident", "prefill", "tiny", "qwen", "trace", "device_fill",
                                    "prefill_layers"],
                   default="all",
                   help="run only that context leg (profiling); prints its own JSON line")
    p.add_argument("--trace-steps", type=int, default=256, help="decode steps of the 40-layer trace leg")
    p.add_argument("--fill", choices=["host", "device"], default="host",
                   help="miss fills of the decode streams: host-issued DMA copies or the zero-copy fill kernel")
    return p.parse_args()


def workload_config(cfg, n, world, fill="host"):
    return {"workload": "DeepSeek-V4-Flash-shaped MXFP4 MoE decode layer: 256 routed experts, top-6, "
                        "hidden 4096, expert FFN 2048, 64-slot GPU expert cache (LRU, misses filled from "
                        "pinned host RAM), Zipf(1.1) routing, continuous decode stream from a cold cache",
            "batch_tokens": n, "experts": cfg.experts, "top_k": cfg.top_k, "hidden": cfg.hidden,
            "ffn": cfg.ffn, "weights": "mxfp4", "activations": "bf16", "capacity_slots": cfg.capacity,
            "routing": "zipf(s=1.1) via router bias, seed 0", "l2": "flushed before every step (256 MiB write)",
            "miss_fills": "zero-copy fill kernel" if fill == "device" else "host-issued DMA copies",
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
    """Dense bf16 tensor peak (burst) and its provenance."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


FP4_OVER_BF16 = 4.0   # nominal dense ratio (9 vs 2.25 PFLOP/s): FP4 peak = bf16 peak x 4


def host_info():
    """CPU model, logical cores and RAM of this host (for the CPU baseline record)."""
    model, mem = "unknown", None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
        for line in open("/proc/meminfo"):
            if line.startswith("MemTotal"):
                mem = int(line.split()[1]) * 1024
                break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count(), "ram_bytes": mem}


class OneCore:
    """Runs the enclosed code pinned to one CPU core (the oracle baseline is single-threaded)."""

    def __enter__(self):
        self.saved = os.sched_getaffinity(0)
        self.core = min(self.saved)
        os.sched_setaffinity(0, {self.core})
        try:
            import torch
            self.threads = torch.get_num_threads()
            torch.set_num_threads(1)
        except ImportError:
            self.threads = None
        return self

    def __exit__(self, *exc):
        os.sched_setaffinity(0, self.saved)
        if self.threads is not None:
            import torch
            torch.set_num_threads(self.threads)
        return False


def measure_bp(device, srcs, mib=64, reps=20):
    """Pinned host -> device copy bandwidth Bp (GB/s): median of `reps` samples, each one
    cudaMemcpyAsync per source buffer until `mib` MiB are copied.  The sources are the
    pinned expert blobs the cache fills from: a fresh pinned buffer can land on another
    NUMA node than the blobs and see a different PCIe path."""
    import torch
    todo, plan = mib << 20, []
    for h in srcs:
        if todo <= 0:
            break
        take = min(todo, h.numel())
        plan.append((h, take))
        todo -= take
    total = sum(t for _, t in plan)
    d = torch.empty(total, dtype=torch.uint8, device=device)

    def once():
        o = 0
        for h, t in plan:
            d[o:o + t].copy_(h[:t], non_blocking=True)
            o += t
    once()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        once()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return total / (float(np.median(ts)) / 1000.0) / 1e9


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

    def __init__(self, cfg, shape, blobs, wg, bias, n, steps, capacity, rank, device, tag="decode", fill="host"):
        import torch

        from expert_cached_sparse_b200 import api as A
        from expert_cached_sparse_b200 import workloads as W
        self.A, self.n, self.cfg, self.shape = A, n, cfg, shape
        self.cache = A.MoeCache(shape, capacity, blobs, trace_capacity=0)
        if fill == "device":
            self.cache.set_fill_mode(1)
        self.wg = to_dev_bits(wg, device)
        self.bias = torch.from_numpy(bias).to(device) if bias is not None else None
        xs = np.stack([W.gen_x(cfg, 1000 + rank, n, tag, s) for s in range(steps)])
        self.x_host = xs
        if cfg.x_dtype == "f32":
            self.x = torch.from_numpy(xs).to(device)          # [steps, n, H] float32
            self.out = torch.empty(n, cfg.hidden, dtype=torch.float32, device=device)
        else:
            self.x = to_dev_bits(xs, device)                  # [steps, n, H] bf16
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


# DRAM bytes (read + write) of the grouped-FFN calls of the headline decode
# stream (one launch of the fused decode kernel per call: the hit pass and
# the miss groups) over their algorithmic bytes, both summed over every call
# of the timed steps of an ncu capture of that workload.  Calls differ in
# size by two orders of magnitude, so the ratio, times this run's
# algorithmic bytes per call, is what is reported per call.  Valid only for
# the FFN code it was measured on (comments aside): other code reports null.
FFN_TRAFFIC = {"source_sha1": "4969e8c3e455cccf8206300e75c7a84d2de318a4", "dram_over_algorithmic": 1.0369}


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


def ffn_traffic(algorithmic_bytes_per_call):
    r = FFN_TRAFFIC["dram_over_algorithmic"]
    if r is None or ffn_source_sha1() != FFN_TRAFFIC["source_sha1"]:
        return None
    return r * algorithmic_bytes_per_call


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
    """A layer step that reads nothing back to the host (every expert resident, or
    device fills) can be captured once in a CUDA graph; replays steps
    first..first+k-1 (inputs copied into the captured input buffer before each,
    outside the events) and returns the summed device ms."""
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
    oracle_token_steps(cfg, 0, min(args.warmup, 2), args.batch)      # warm-up samples
    with OneCore() as oc:
        sec, toks = oracle_token_steps(cfg, 0, args.steps, args.batch)
    value = toks / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sec / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg, args.batch, world, args.fill),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "pinned_core": oc.core, **host_info(),
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
                     batches=tuple(int(b) for b in args.resident_batch.split(",")), trace_steps=args.trace_steps,
                     cpu=not args.no_cpu_baseline, fill=args.fill)
        if rank == 0:
            print(json.dumps({"leg": args.leg, "steps": K, "warmup": Wm, "results": res}), flush=True)
        return

    # ---- headline: 64-slot decode stream
    distinct_blobs = list({b.data_ptr(): b for b in blobs}.values())
    bp0 = measure_bp(device, distinct_blobs)
    ds = DecodeStream(cfg, shape, blobs, wg, bias, n, 2 * K + Wm, cfg.capacity, rank, device, fill=args.fill)
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
            "dtype": "bf16", "data": "synthetic", "config": workload_config(cfg, n, world, args.fill)}
    line["roofline"] = {"kernel": "grouped SwiGLU FFN call (ffn_fp4_fused_kernel: x terms, gate-up, h terms, "
                                  "down; block-scaled tcgen05)",
                        "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                        "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                        "traffic": ffn_traffic(ffn_bytes / ffn_calls),
                        "algorithmic_bytes_per_call": ffn_bytes / ffn_calls,
                        "avg_call_ms": ffn_ms / ffn_calls, "calls": ffn_calls}
    # Bp before and after the timed region (the PCIe path can be shared with
    # other traffic on the host); the bound takes the better of the two
    bp1 = measure_bp(device, distinct_blobs)
    bp = max(bp0, bp1)
    # the step's end-to-end bound: its HBM bytes at the measured peak plus its misses over PCIe at Bp
    step_hbm = ffn_bytes / K + cfg.experts * cfg.hidden * 2 + 2 * n * cfg.hidden * 2
    bound_ms = step_hbm / (hbm_peak * 1e9) * 1e3 + (misses / K) * slot_bytes / (bp * 1e9) * 1e3
    line["bp_GBps"] = bp
    line["bp_GBps_before_after"] = [bp0, bp1]
    line["step_bound"] = {"ms_per_step": bound_ms, "frac": bound_ms / (ms_max / K),
                          "note": "HBM bytes of the step at the measured peak + misses x slot bytes / Bp "
                                  "(Bp: 64 MiB of the pinned expert blobs copied host->device, median of 20, measured "
                                  "before and after the timed steps in this run, the better taken)"}
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
        line["extras"] = extras(cfg, shape, blobs, wg, bias, K, Wm, flush, device, hbm_peak,
                                trace_steps=args.trace_steps, cpu=world == 1 and not args.no_cpu_baseline,
                                fill=args.fill)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with OneCore() as oc:
            sec, toks = oracle_token_steps(cfg, 0, 16, n)
        line["cpu_baseline"] = {"value": toks / sec, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "pinned_core": oc.core, **host_info(),
                                "sample": f"{toks} one-token samples of the same decode stream (route, LRU, "
                                          f"dequantise 6 experts, 6 SwiGLU FFNs, combine), "
                                          f"{sec:.1f} s on one pinned core"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def pinned_blobs(cfg, seed, distinct=None):
    """Pinned packed blobs of every (layer, expert) key; with `distinct`, keys share that many weight sets."""
    import torch

    from expert_cached_sparse_b200 import api as A
    from expert_cached_sparse_b200 import workloads as W
    shape = A.shape_of(cfg)
    sb = A.moe_slot_bytes(shape)
    made, blobs = {}, []
    for l in range(cfg.layers):
        for e in range(cfg.experts):
            key = W.blob_alias(cfg, l, e, distinct)
            if key not in made:
                b = torch.empty(sb, dtype=torch.uint8, pin_memory=True)
                A.moe_pack_expert(shape, W.gen_expert(cfg, seed, *key), out=b.numpy())
                made[key] = b
            blobs.append(made[key])
    return shape, blobs


def oracle_rate(cfg, seed, xs, wg, bias, expert_fn, layers=None):
    """The CPU oracle, pinned to one core, on the token samples xs (list of [n, H] arrays, one per layer
    call): seconds and tokens.  Expert weights are inputs, generated before the clock starts."""
    from oracle import oracle as O
    O.build()
    for i, x in enumerate(xs):
        _, idx, _ = O.router(x, wg[i] if isinstance(wg, list) else wg,
                             (bias[i] if isinstance(bias, list) else bias), cfg.top_k)
        for e in np.unique(idx):
            expert_fn(i, int(e))
    with OneCore() as oc:
        t0 = time.perf_counter()
        toks = 0
        for i, x in enumerate(xs):
            O.moe_layer(x, wg[i] if isinstance(wg, list) else wg, bias[i] if isinstance(bias, list) else bias,
                        cfg.top_k, cfg.wfmt, cfg.hidden, cfg.ffn, lambda e, i=i: expert_fn(i, e))
            toks += x.shape[0]
        sec = time.perf_counter() - t0
        core = oc.core
    return sec, toks, core


def cpu_line(value, sec, toks, core, sample):
    return {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "pinned_core": core,
            "sample": f"{sample}; {toks} tokens in {sec:.1f} s", **host_info()}


def layer_leg(cfg, shape, blobs, wg, bias, n, steps, warm, flush, device, hbm_peak, tag, capacity=None,
              graph=True):
    """Fully resident single-layer steps of n tokens: per-step ms (eager and CUDA-graph replay), the
    FFN's HBM fraction, the layer's HBM fraction and the step breakdown."""
    import torch

    from expert_cached_sparse_b200 import api as A
    slot_bytes = A.moe_slot_bytes(shape)
    ds = DecodeStream(cfg, shape, blobs, wg, bias, n, steps + warm, capacity or cfg.experts, 0, device, tag=tag)
    ds.cache.lookup_update(0, torch.arange(cfg.experts, dtype=torch.int32, device=device))
    torch.cuda.synchronize()
    for s in range(warm):
        ds.step(s)
    torch.cuda.synchronize()
    A.moe_profile_read(reset=True)
    A.moe_profile_enable(True)
    ms = timed_steps(ds, warm, steps, flush, False)
    prof = A.moe_profile_read(reset=True)
    A.moe_profile_enable(False)
    idx = ds.idx[warm:warm + steps].cpu().numpy()
    fb = ffn_algorithmic_bytes(idx, cfg, slot_bytes)
    layer_bytes = fb + steps * (cfg.experts * cfg.hidden * 2 + 2 * n * cfg.hidden * (4 if cfg.x_dtype == "f32" else 2))
    ffn_s = prof["ffn"]["ms"] / 1000
    out = {"tokens": n, "tokens_per_s": steps * n / (ms / 1000), "ms_per_step": ms / steps,
           "layer_hbm_frac": layer_bytes / (ms / 1000) / 1e9 / hbm_peak,
           "ffn_ms_per_step": prof["ffn"]["ms"] / steps,
           "ffn_GBps": fb / ffn_s / 1e9, "ffn_hbm_frac": fb / ffn_s / 1e9 / hbm_peak,
           "unique_experts_per_step": float(np.mean([len(np.unique(i)) for i in idx])),
           "step_ms_breakdown": {k: prof[k]["ms"] / steps for k in prof}}
    if graph:
        gms = graph_steps(ds, warm, steps, flush)
        out["cuda_graph"] = {"tokens_per_s": steps * n / (gms / 1000), "ms_per_step": gms / steps,
                             "note": "the same resident steps captured once in a CUDA graph and replayed "
                                     "(one replay per step, L2 flushed before each, profiling off)"}
    ds.cache.close()
    return out, ds.x_host


def prefill_layers_leg(device, nl=4, n=4096, distinct=24, reps=2):
    """4096 tokens through 4 DeepSeek-shaped MXFP4 layers (each with its own input), cold cache: with 512 slots the next layer's 256 experts stream in over PCIe while the current layer
    computes; with 256 slots (one layer) its fills follow the compute.  Compute alone is timed on a
    warm 1024-slot cache (every lookup hits).  Host blobs aliased to `distinct` weight sets."""
    import torch

    from expert_cached_sparse_b200 import api as A
    from expert_cached_sparse_b200 import workloads as W
    cfg = W.scaled(W.DS_PREFILL, layers=nl)
    E = cfg.experts
    shape, blobs = pinned_blobs(cfg, 0, distinct)
    sb = A.moe_slot_bytes(shape)
    bp = measure_bp(device, list({b.data_ptr(): b for b in blobs}.values()))
    wgs = [to_dev_bits(W.gen_wg(cfg, 0, l), device) for l in range(nl)]
    biases = [torch.from_numpy(W.gen_bias(cfg, 0, l, 0)).to(device) for l in range(nl)]
    xs = [to_dev_bits(W.gen_x(cfg, 0, n, "prefill", l), device) for l in range(nl)]
    outs = [torch.empty_like(xs[0]) for _ in range(nl)]
    ws = torch.empty(A.moe_prefill_workspace_bytes(shape, n), dtype=torch.uint8, device=device)
    st, cp = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def run(cache):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(st)
        A.moe_prefill_forward(cache, 0, xs, wgs, biases, outs, ws, stream=st, copy_stream=cp)
        b.record(st)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    out = {"layers": nl, "tokens": n, "bp_GBps": bp, "layer_fill_bytes": E * sb, "host_blob_sets": distinct}
    warm = A.MoeCache(shape, nl * E, blobs, trace_capacity=0)
    run(warm)
    compute_ms = min(run(warm) for _ in range(reps))
    warm.close()
    del warm
    out["compute_ms"] = compute_ms
    for name, cap in (("double_buffered_512_slots", 2 * E), ("one_layer_256_slots", E)):
        ts = []
        for _ in range(reps):
            cache = A.MoeCache(shape, cap, blobs, trace_capacity=0)
            ts.append(run(cache))
            cache.close()
            del cache
        out[name] = {"ms": min(ts), "tokens_per_s": n / (min(ts) / 1000)}
    fill_ms = E * sb / (bp * 1e9) * 1e3
    layer_ms = compute_ms / nl
    # the first layer's fills precede any compute; then each layer's fills hide the previous
    # layer's compute (or the reverse); the last layer computes alone
    pipe_ms = fill_ms + (nl - 1) * max(fill_ms, layer_ms) + layer_ms
    out["bound"] = {"per_layer_ms": max(layer_ms, fill_ms), "pipeline_ms": pipe_ms,
                    "sequential_ms": nl * (fill_ms + layer_ms),
                    "note": "per layer max(compute, layer bytes / Bp); pipeline = fill + (L-1) max(fill, "
                            "compute) + compute; sequential = L (fill + compute)"}
    out["double_buffered_512_slots"]["frac_of_pipeline_bound"] = pipe_ms / out["double_buffered_512_slots"]["ms"]
    out["one_layer_256_slots"]["frac_of_sequential_bound"] = out["bound"]["sequential_ms"] / \
        out["one_layer_256_slots"]["ms"]
    del blobs
    return out


def device_fill_leg(cfg, shape, blobs, wg, bias, n, K, Wm, flush, device):
    """The headline decode stream (cold 64-slot cache) with device fills: eager calls, then
    a fresh cache whose whole step, misses included, is one CUDA graph replayed per step."""
    import torch
    out = {}
    for mode in ("eager", "cuda_graph"):
        ds = DecodeStream(cfg, shape, blobs, wg, bias, n, K + Wm, cfg.capacity, 0, device, fill="device")
        for s in range(Wm):
            ds.step(s)
        torch.cuda.synchronize()
        st0 = ds.cache.stats()
        ms = timed_steps(ds, Wm, K, flush, False) if mode == "eager" else graph_steps(ds, Wm, K, flush)
        st1 = ds.cache.stats()
        misses = st1["misses"] - st0["misses"]
        hits = st1["hits"] - st0["hits"]
        out[mode] = {"tokens_per_s": K * n / (ms / 1000), "ms_per_step": ms / K,
                     "hit_rate": hits / max(1, hits + misses), "misses_per_step": misses / K,
                     "host_syncs": st1["host_syncs"] - st0["host_syncs"]}
        ds.cache.close()
        del ds
    out["note"] = ("misses copied by the zero-copy fill kernel from mapped pinned blobs; nothing is read back, "
                   "so the graph holds the whole step; L2 flushed before each step")
    return out


def extras(cfg, shape, blobs, wg, bias, K, Wm, flush, device, hbm_peak, legs=("resident", "prefill", "tiny", "qwen",
                                                                              "trace", "device_fill",
                                                                              "prefill_layers"),
           batches=(1, 4, 16), trace_steps=256, cpu=True, fill="host"):
    """Context legs: every other workload of the layer, each with its roofline fraction and the oracle's
    single-core rate on a bounded sample."""
    import torch

    from expert_cached_sparse_b200 import api as A
    from expert_cached_sparse_b200 import workloads as W
    out = {}
    tensor_peak, tensor_kind = measured_bf16_tflops()
    # ---- multi-layer prefill with full-layer double buffering
    if "prefill_layers" in legs:
        out["prefill_4x4096_double_buffered"] = prefill_layers_leg(device)
    # ---- the headline stream with device-initiated fills
    if "device_fill" in legs:
        out["decode_b16_device_fill"] = device_fill_leg(cfg, shape, blobs, wg, bias, 16, K, Wm, flush, device)
    # ---- the DeepSeek-shaped MXFP4 layer, every expert resident (decode, HBM-bound)
    for n in (batches if "resident" in legs else ()):
        r, _ = layer_leg(cfg, shape, blobs, wg, bias, n, K, Wm, flush, device, hbm_peak, "resident")
        out[f"resident_decode_b{n}"] = r
    # ---- its 4096-token prefill (Zipf 0.8, all experts resident)
    if "prefill" in legs:
        pcfg = W.DS_PREFILL
        pbias = W.gen_bias(pcfg, 0, 0)
        steps = 3
        r, xh = layer_leg(pcfg, shape, blobs, wg, pbias, 4096, steps, 1, flush, device, hbm_peak, "prefill",
                          graph=False)
        flops = 4096 * cfg.top_k * 3 * 2 * cfg.hidden * cfg.ffn
        ffn_s = r["ffn_ms_per_step"] / 1000
        r["ffn_tflops_bf16_equiv"] = flops / ffn_s / 1e12
        r["ffn_bf16_frac"] = flops / ffn_s / 1e12 / tensor_peak
        r["ffn_fp4_peak_frac"] = flops / ffn_s / 1e12 / (tensor_peak * FP4_OVER_BF16)
        r["ffn_fp4_pipe_frac"] = 3 * flops / ffn_s / 1e12 / (tensor_peak * FP4_OVER_BF16)
        r["tensor_peak_tflops_bf16"] = tensor_peak
        r["tensor_peak_kind"] = tensor_kind
        r["note"] = ("FP4 peak = bf16 peak x 4 (nominal ratio); fp4_pipe_frac counts the 3 E2M1 activation "
                     "terms the prefill tiles multiply")
        if cpu:
            experts = {}

            def efn(i, e):
                if e not in experts:
                    experts[e] = W.gen_expert(pcfg, 0, 0, e)
                return experts[e]
            sec, toks, core = oracle_rate(pcfg, 0, [xh[1][:8]], wg, pbias, efn)
            r["cpu_baseline"] = cpu_line(toks / sec, sec, toks, core,
                                         "8 tokens of the 4096-token prefill batch, scaled per token")
        out["prefill_4096"] = r
    # ---- the tiny BF16 layer (64 tokens, 8 experts, fp32 activations): launch-bound
    if "tiny" in legs:
        tcfg = W.TINY
        tshape, tblobs = pinned_blobs(tcfg, 0)
        twg, tb = W.gen_wg(tcfg, 0, 0), None
        r, xh = layer_leg(tcfg, tshape, tblobs, twg, tb, 64, 20, 3, flush, device, hbm_peak, "tiny")
        r["bound"] = "launch latency (6.3 MB of weights)"
        if cpu:
            texperts = {e: W.gen_expert(tcfg, 0, 0, e) for e in range(tcfg.experts)}
            sec, toks, core = oracle_rate(tcfg, 0, [xh[0]], twg, tb, lambda i, e: texperts[e])
            r["cpu_baseline"] = cpu_line(toks / sec, sec, toks, core, "one full 64-token call")
        out["tiny_64"] = r
    # ---- the Qwen-shaped BF16 layer: 512-token prefill and 8-token decode batches (HBM-bound)
    if "qwen" in legs:
        qcfg = W.QWEN_BF16
        qshape, qblobs = pinned_blobs(qcfg, 0)
        qwg = W.gen_wg(qcfg, 0, 0)
        r, xh = layer_leg(qcfg, qshape, qblobs, qwg, None, 512, 5, 2, flush, device, hbm_peak, "qwen-prefill",
                          graph=False)
        qexperts = {}

        def qfn(i, e):
            if e not in qexperts:
                qexperts[e] = W.gen_expert(qcfg, 0, 0, e)
            return qexperts[e]
        if cpu:
            sec, toks, core = oracle_rate(qcfg, 0, [xh[2][:8]], qwg, None, qfn)
            r["cpu_baseline"] = cpu_line(toks / sec, sec, toks, core,
                                         "8 tokens of the 512-token prefill batch, scaled per token")
        out["qwen_prefill_512"] = r
        r, xh = layer_leg(qcfg, qshape, qblobs, qwg, None, 8, 64, 3, flush, device, hbm_peak, "qwen-decode")
        if cpu:
            sec, toks, core = oracle_rate(qcfg, 0, [xh[3]], qwg, None, qfn)
            r["cpu_baseline"] = cpu_line(toks / sec, sec, toks, core, "one 8-token decode batch")
        out["qwen_decode_8"] = r
        del qblobs
    # ---- the 40-layer NVFP4 decode trace: shared 1024-slot cache, misses filled over PCIe
    if "trace" in legs:
        out["trace40"] = trace_leg(trace_steps, flush, device, hbm_peak, cpu, fill=fill)
    return out


def trace_leg(steps, flush, device, hbm_peak, cpu=True, distinct=64, fill="host"):
    """256 one-token decode steps through 40 NVFP4 layers (per-layer Zipf(1.0) routing with 10% rank
    drift every 32 steps) sharing one 1024-slot cache, cold; misses filled from pinned host RAM.
    Host blobs are aliased to `distinct` weight sets (cache behaviour does not depend on contents)."""
    import torch

    from expert_cached_sparse_b200 import api as A
    from expert_cached_sparse_b200 import workloads as W
    cfg = W.TRACE40
    shape, blobs = pinned_blobs(cfg, 0, distinct)
    sb = A.moe_slot_bytes(shape)
    cache = A.MoeCache(shape, cfg.capacity, blobs, trace_capacity=0)
    if fill == "device":
        cache.set_fill_mode(1)
    wgs = [to_dev_bits(W.gen_wg(cfg, 0, l), device) for l in range(cfg.layers)]
    nep = (steps + cfg.drift_every - 1) // cfg.drift_every
    biases = {(l, ep): torch.from_numpy(W.gen_bias(cfg, 0, l, ep)).to(device)
              for l in range(cfg.layers) for ep in range(nep)}
    xs = to_dev_bits(np.stack([W.gen_x(cfg, 2000, 1, "trace", s) for s in range(steps)]), device)
    out_t = torch.empty(1, cfg.hidden, dtype=torch.bfloat16, device=device)
    ws = torch.empty(A.moe_layer_workspace_bytes(shape, 1), dtype=torch.uint8, device=device)
    st, cp = torch.cuda.Stream(device), torch.cuda.Stream(device)
    idx = torch.empty(steps, cfg.layers, cfg.top_k, dtype=torch.int32, device=device)
    torch.cuda.synchronize()
    st0 = cache.stats()
    A.moe_profile_read(reset=True)
    A.moe_profile_enable(True)
    evs = []
    for s in range(steps):
        with torch.cuda.stream(st):
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        ep = W.drift_epoch(cfg, s)
        for l in range(cfg.layers):
            A.moe_layer_forward(cache, l, xs[s], wgs[l], biases[(l, ep)], out_t, ws, stream=st, copy_stream=cp,
                                topk_idx_out=idx[s, l])
        b.record(st)
        evs.append((a, b))
    torch.cuda.synchronize()
    prof = A.moe_profile_read(reset=True)
    A.moe_profile_enable(False)
    st1 = cache.stats()
    ms = sum(a.elapsed_time(b) for a, b in evs)
    hits, misses = st1["hits"] - st0["hits"], st1["misses"] - st0["misses"]
    fill_bytes = st1["fill_bytes"] - st0["fill_bytes"]
    fill_ms = prof["fill"]["ms"]
    # compute segments: each layer call's FFN streams its 6 experts' weights
    ffn_bytes = steps * cfg.layers * (cfg.top_k * sb) + steps * cfg.layers * cfg.top_k * (cfg.hidden + cfg.ffn) * 4
    ffn_s = prof["ffn"]["ms"] / 1000
    r = {"steps": steps, "layers": cfg.layers, "tokens_per_s": steps / (ms / 1000), "ms_per_token": ms / steps,
         "hit_rate": hits / max(1, hits + misses), "misses_per_token": misses / steps,
         "fill_GBps": fill_bytes / (fill_ms / 1000) / 1e9 if fill_ms > 0 else None,
         "ffn_hbm_frac": ffn_bytes / ffn_s / 1e9 / hbm_peak if ffn_s > 0 else None,
         "all_hit_bound_ms_per_token": cfg.layers * (2 * 1024 * 1024 + cfg.top_k * sb) / (hbm_peak * 1e9) * 1e3,
         "host_blob_sets": distinct, "step_ms_breakdown": {k: prof[k]["ms"] / steps for k in prof}}
    cache.close()
    if cpu:
        experts = {}

        def efn(i, e):
            key = W.blob_alias(cfg, i, e, distinct)
            if key not in experts:
                experts[key] = W.gen_expert(cfg, 0, *key)
            return experts[key]
        xs_h = [W.gen_x(cfg, 2000, 1, "trace", 0)] * 2
        wgl = [W.gen_wg(cfg, 0, l) for l in range(2)]
        bl = [W.gen_bias(cfg, 0, l, 0) for l in range(2)]
        sec, toks, core = oracle_rate(cfg, 0, xs_h, wgl, bl, efn)
        tok_s = 1.0 / (sec / 2 * cfg.layers)     # one token = 40 layer calls
        r["cpu_baseline"] = cpu_line(tok_s, sec, toks, core,
                                     "one token through 2 of the 40 layers, scaled to 40 layers")
    del blobs
    return r


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
