#!/usr/bin/env python
"""Benchmark of the heterogeneous-batch LoRA adapter branch on B200.

Metric: LoRA-branch tokens/s per layer.  One step = one batch through the
whole hot path: the segment plan of the batch (made once, as a model does for
all of its adapted layers) and the fused shrink + expand-add of every layer
in a ring of independent layer instances (own pools, page tables, X and Y per
layer).  The ring's footprint is more than 4x the L2 cache, so every layer's
weights and activations come from HBM.  The step is captured once in a CUDA
graph and replayed.  value = tokens x layers x steps / device time.

Default (headline) workload: the largest single-GPU configuration, the 8B
sweep with every token on a distinct adapter at T = 1024 (d_in = 4096,
d_out = 14336, rank 64, 512 resident adapters, 1.33 GB of algorithmic bytes
per layer).  The same JSON line carries `per_config`: kernel time, algorithmic
bytes and the fraction of the measured HBM peak for every other configuration
(7B decode q_proj, mixed-rank MLP up and down, prefill with its tensor-pipe
fraction, the 8B sweep at T = 1, 64, 1024 in both regimes).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LoRA-branch tokens/s per layer"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="sweep_8b_distinct_T1024",
                   help="decode_q_proj_7b | mixed_mlp_up | mixed_mlp_down | prefill | sweep_8b_one_T<n> | sweep_8b_distinct_T<n>")
    p.add_argument("--layers", type=int, default=0, help="ring size (0 = enough for > 4x L2)")
    p.add_argument("--projections", type=int, default=1,
                   help="layers that share one X and one launch (lora_apply_multi_planned), e.g. 3 for q/k/v")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-config", action="store_true")
    p.add_argument("--no-prefetch", action="store_true")
    p.add_argument("--per-config", default=",".join(PER_CONFIG),
                   help="comma-separated workloads measured into the per_config object")
    return p.parse_args()


# Every configuration of the workload list; the headline is the largest.
PER_CONFIG = ["decode_q_proj_7b", "mixed_mlp_up", "mixed_mlp_down", "prefill",
              "sweep_8b_one_T1", "sweep_8b_one_T64", "sweep_8b_one_T1024",
              "sweep_8b_distinct_T1", "sweep_8b_distinct_T64", "sweep_8b_distinct_T1024"]


# ---------------------------------------------------------------------------
# Workload description (shapes and ids only; weights are drawn per layer)
# ---------------------------------------------------------------------------

def workload_spec(name: str):
    import workloads as W
    if name == "decode_q_proj_7b":
        wl = W.decode_q_proj_7b()
        desc = ("7B decode q_proj: d_in=d_out=4096, 64 tokens (1/seq), 32 resident rank-16 adapters "
                "drawn Zipf(1.0) from a 1000-adapter catalogue, bf16 weights in 16-row pages, fp32 Y_base")
    elif name in ("mixed_mlp_up", "mixed_mlp_down"):
        wl = W.mixed_mlp(which=name.split("_")[-1])
        desc = f"mixed-rank decode MLP {name.split('_')[-1]}: 256 tokens, 128 resident adapters r in {{8,16,32,64}}, Zipf(1.1)"
    elif name == "prefill":
        wl = W.prefill()
        desc = "prefill: 16 sequences of 128-2048 tokens, d=4096, 6 adapters r in {8,16,32,64}"
    elif name.startswith("sweep_8b_"):
        _, _, regime, tt = name.split("_")
        wl = W.sweep_8b(T=int(tt[1:]), regime=regime)
        desc = f"8B sweep {regime}: d_in=4096, d_out=14336, rank 64, pool of 512, T={tt[1:]}"
    else:
        raise SystemExit(f"unknown workload {name}")
    return wl, desc


def algorithmic_bytes(wl) -> int:
    """Each distinct adapter read once (A and B, bf16), X read in bf16, Y read and written in fp32,
    over the tokens whose slot holds an adapter."""
    ids = wl.ids
    rk = wl.ranks()
    inr = (ids >= 0) & (ids < wl.S)
    valid = ids[inr][rk[ids[inr]] > 0]
    distinct = np.unique(valid)
    w = int(sum(2 * int(rk[i]) * (wl.d_in + wl.d_out) for i in distinct))
    return w + len(valid) * (2 * wl.d_in + 8 * wl.d_out)


def algorithmic_flops(wl) -> int:
    ids = wl.ids
    rk = wl.ranks()
    inr = (ids >= 0) & (ids < wl.S)
    valid = ids[inr][rk[ids[inr]] > 0]
    return int(sum(2 * int(rk[i]) * (wl.d_in + wl.d_out) for i in valid))


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
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
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def time_oracle(wl, seconds: float, max_flops: float = 2.5e8):
    """Run the fp64 C oracle on the workload's batch until `seconds` of work
    (at least one call); returns (tokens/s per layer, threads, sample text)."""
    from oracle import build_oracle as OC
    T = wl.T
    # bounded sample: whole batch when small, else the first tokens of it
    n_tok = T
    est = algorithmic_flops(wl)
    if est > max_flops:
        n_tok = max(1, int(T * max_flops / est))
    tok = np.arange(n_tok)
    import workloads as W
    X, Yb, ids, A, B, sc = W.subset_for_tokens(wl, tok)
    threads = OC.max_threads()
    calls = 0
    t0 = time.perf_counter()
    while True:
        OC.lora_apply_c(X, Yb, ids, A, B, sc, nthreads=threads)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    value = n_tok * calls / el
    sample = f"{calls} oracle calls of {n_tok} tokens ({wl.name}), {el:.1f} s"
    return value, threads, sample


def ring_layers(wl, layers_arg: int = 0, factor: float = 4.2) -> int:
    """Independent layer instances so that one step's footprint exceeds factor x L2."""
    per_layer = (wl.pages_a * 16 * wl.d_in * 2 + wl.pages_b * 16 * wl.d_out * 2
                 + wl.T * (wl.d_in * 2 + wl.d_out * 4))
    return layers_arg or max(8, min(256, math.ceil(factor * L2_BYTES / per_layer)))


def bench_config(wl, desc: str, layers_arg: int = 0) -> dict:
    """The workload's config object, identical on both arms."""
    n = ring_layers(wl, layers_arg)
    return {"workload": desc, "tokens": wl.T, "distinct_adapters": wl.distinct(),
            "l2": f"inputs larger than L2: a ring of {n} independent layer instances "
                  f"(over 4 x the 126 MB L2) replayed back to back"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl, desc = workload_spec(args.workload)
    # one step = oracle calls on the workload's batch (its first tokens when the
    # batch is large) for at least 20 ms; the value is the median step rate
    per_step = []
    for _ in range(max(args.warmup, 0)):
        time_oracle(wl, 0.02)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, threads, sample = time_oracle(wl, 0.02)
        per_step.append(v)
    el = time.perf_counter() - t0
    value = statistics.median(per_step)
    sample = f"{args.steps} steps, each {sample}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * el / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, desc),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class Ring:
    """L independent layer instances sharing one batch (ids, plan)."""

    def __init__(self, wl, n_layers: int, seed: int, device):
        import torch
        import heterogeneous_adapter_batching_b200 as H
        self.H = H
        self.wl = wl
        self.T = wl.T
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        ranks = wl.ranks()
        self.layers, self.X, self.Y = [], [], []
        for l in range(n_layers):
            lay = H.AdapterLayer(wl.d_in, wl.d_out, wl.S, wl.pages_a, wl.pages_b, wl.T, device=device)
            for i in range(wl.S):
                r = int(ranks[i])
                if r <= 0:
                    continue
                at = (torch.randn((r, wl.d_in), generator=g, device=device) / math.sqrt(wl.d_in)).to(torch.bfloat16)
                b = (torch.randn((r, wl.d_out), generator=g, device=device) / math.sqrt(r)).to(torch.bfloat16)
                lay.load(i, r, float(wl.adapters.alpha_of[i]), at, b,
                         page_ids=torch.from_numpy(np.ascontiguousarray(wl.page_ids[i])))
            self.layers.append(lay)
            self.X.append((torch.randn((wl.T, wl.d_in), generator=g, device=device) / math.sqrt(wl.d_in)).to(torch.bfloat16))
            self.Y.append(torch.randn((wl.T, wl.d_out), generator=g, device=device))
        self.ids = torch.from_numpy(wl.ids.copy()).to(device)
        self.ws = torch.empty(H.lora_workspace_size(wl.T, wl.S), dtype=torch.uint8, device=device)
        torch.cuda.synchronize()

    def footprint(self) -> int:
        lay = self.layers[0]
        per = (lay.buf_a.numel() * 2 + lay.buf_b.numel() * 2 + self.X[0].numel() * 2 + self.Y[0].numel() * 4)
        return per * len(self.layers)

    def step(self, stream=None) -> int:
        """Plan once, apply every layer; returns the number of kernels launched."""
        H = self.H
        lay0 = self.layers[0]
        lay0.plan(self.ids, ws=self.ws, stream=stream)
        n = H.lora_last_launch_count()
        for lay, X, Y in zip(self.layers, self.X, self.Y):
            lay.apply_planned(X, Y, ws=self.ws, stream=stream)
            n += H.lora_last_launch_count()
        return n

    def apply_only(self, stream=None) -> int:
        n = 0
        for lay, X, Y in zip(self.layers, self.X, self.Y):
            lay.apply_planned(X, Y, ws=self.ws, stream=stream)
            n += self.H.lora_last_launch_count()
        return n

    def step_groups(self, P: int, stream=None, plan: bool = True) -> int:
        """Plan once, then one lora_apply_multi_planned per group of P layers that
        read the same X (the group's first); returns the number of kernels launched."""
        H = self.H
        n = 0
        if plan:
            self.layers[0].plan(self.ids, ws=self.ws, stream=stream)
            n += H.lora_last_launch_count()
        for g in range(0, len(self.layers), P):
            H.apply_multi(self.layers[g:g + P], self.X[g], self.Y[g:g + P], None, ws=self.ws, stream=stream)
            n += H.lora_last_launch_count()
        return n

    def plan_only(self, reps: int, stream=None) -> int:
        """The batch's plan, `reps` times (timing of the plan kernel)."""
        n = 0
        for _ in range(reps):
            self.layers[0].plan(self.ids, ws=self.ws, stream=stream)
            n += self.H.lora_last_launch_count()
        return n

    def apply_calls(self, reps: int, stream=None) -> int:
        """lora_apply (plan + compute in one call) on the first min(reps, layers) layers."""
        n = 0
        for lay, X, Y in list(zip(self.layers, self.X, self.Y))[:reps]:
            self.H.lora_apply(X, Y, self.T, lay.d_in, lay.d_out, self.ids, lay.S, lay.ranks, lay.scales,
                              lay.page_table, lay.pool_a, lay.pool_b, self.ws, lay.err, stream)
            n += self.H.lora_last_launch_count()
        return n

    def step_groups_separate(self, P: int, stream=None) -> int:
        """The same work as step_groups(plan=False) with one launch per layer."""
        n = 0
        for g in range(0, len(self.layers), P):
            for lay, Y in zip(self.layers[g:g + P], self.Y[g:g + P]):
                lay.apply_planned(self.X[g], Y, ws=self.ws, stream=stream)
                n += self.H.lora_last_launch_count()
        return n


# workload -> profile summary of its dominant kernel (each names the kernel source it was captured from)
PROFILE_FOR = {
    "sweep_8b_distinct_T1024": "profiles/split_kernels_sweep_8b_distinct_T1024.md",
    "decode_q_proj_7b": "profiles/gather_kernel_decode_q_proj_7b.md",
    "mixed_mlp_up": "profiles/gather_kernel_mixed_mlp_up.md",
    "prefill": "profiles/tiles_kernels_prefill.md",
    "sweep_8b_one_T1024": "profiles/tiles_kernels_sweep_8b_one_T1024.md",
}


def source_digest(path: str) -> str:
    """sha256 of a CUDA source with its comments and blank lines removed, so that
    a comment-only edit keeps the digest of the code a profile was taken from."""
    import hashlib
    import re
    text = open(path, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def profile_fields(prof_rel: str) -> dict:
    fields = {}
    for line in open(os.path.join(ROOT, prof_rel)):
        if ":" in line and not line.startswith(("#", "|", " ")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    return fields


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when there is none or the kernel's code changed since the capture."""
    if workload not in PROFILE_FOR:
        return None
    try:
        f = profile_fields(PROFILE_FOR[workload])
        if f.get("source_digest") != source_digest(os.path.join(ROOT, f["source"])):
            return None
        return int(f["traffic_bytes_per_launch"])
    except Exception:
        return None


def measured_peaks():
    """(HBM GB/s, bf16 TFLOP/s sustained, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        tf = d.get("bf16_tflops_sustained", d.get("bf16_tflops"))
        return float(d["hbm_gbs"]), float(tf), "measured"
    except Exception:
        return 6650.0, 1400.0, "fallback"


def _time_graph(graph, reps: int, stream) -> float:
    """Mean ms per replay of a captured graph, CUDA events on the replay stream."""
    import torch
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    e0.record(cur)
    for _ in range(reps):
        graph.replay()
    e1.record(cur)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def _capture(fn, stream):
    import torch
    with torch.cuda.stream(stream):
        fn(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        n = fn(stream)
    torch.cuda.synchronize()
    return g, n


def kernel_times(ring, stream, reps: int, H, P: int = 1):
    """Per-layer device times, at the library's default options, of the ring's
    compute launches (the plan already in ring.ws), of the plan alone, and of one
    lora_apply call (plan + compute)."""
    n_valid, n_seg, n_jobs, n_tiles = (int(x) for x in ring.ws[:16].cpu().numpy().view(np.int32)[:4])
    fn = ring.apply_only if P == 1 else (lambda s: ring.step_groups(P, s, plan=False))
    g_apply, launches = _capture(fn, stream)
    n_layers = len(ring.layers)
    apply_ms = _time_graph(g_apply, reps, stream)
    g_plan, _ = _capture(lambda s: ring.plan_only(8, s), stream)
    plan_ms = _time_graph(g_plan, reps, stream) / 8
    g_one, _ = _capture(lambda s: ring.apply_calls(8, s), stream)
    one_ms = _time_graph(g_one, reps, stream) / min(8, n_layers)
    del g_apply, g_plan, g_one
    ring.layers[0].plan(ring.ids, ws=ring.ws, stream=stream)
    torch_sync()
    return {"kernel_us": apply_ms * 1000.0 / n_layers, "plan_us": plan_ms * 1000.0,
            "lora_apply_us": one_ms * 1000.0, "launches_per_layer": launches / n_layers,
            "gather_jobs": n_jobs, "tensor_tiles": n_tiles}


def torch_sync():
    import torch
    torch.cuda.synchronize()


def measure_config(name: str, dev, stream, H, reps: int, peak_gbs: float, peak_tf: float) -> dict:
    """One per_config entry: a ring over 2.5 x L2, the plan once, the compute launches timed."""
    import torch
    wl, desc = workload_spec(name)
    ring = Ring(wl, ring_layers(wl, 0, factor=2.5), seed=4321, device=dev)
    with torch.cuda.stream(stream):
        ring.layers[0].plan(ring.ids, ws=ring.ws, stream=stream)
    torch.cuda.synchronize()
    kt = kernel_times(ring, stream, reps, H)
    alg = algorithmic_bytes(wl)
    flops = algorithmic_flops(wl)
    us = kt["kernel_us"]
    out = {"tokens": wl.T, "distinct_adapters": wl.distinct(), "layers": len(ring.layers),
           "kernel_us": us, "algorithmic_bytes": alg, "achieved_gbs": alg / (us * 1e-6) / 1e9,
           "frac": alg / (us * 1e-6) / 1e9 / peak_gbs, "tokens_per_s": wl.T / (us * 1e-6),
           "plan_us": kt["plan_us"], "lora_apply_us": kt["lora_apply_us"],
           "launches_per_layer": kt["launches_per_layer"],
           "plan": {"gather_jobs": kt["gather_jobs"], "tensor_tiles": kt["tensor_tiles"]}}
    if kt["tensor_tiles"] > 0:
        out["tensor_tflops"] = flops / (us * 1e-6) / 1e12
        out["tensor_frac"] = out["tensor_tflops"] / peak_tf
    del ring
    torch.cuda.empty_cache()
    return out


def measure_prefetch(dev, H, graph, stream, n_adapters: int = 32, d_in: int = 4096, d_out: int = 14336,
                     rank: int = 64) -> dict:
    """Asynchronous adapter loads into a paged pool (AdapterPrefetcher, pinned host
    memory, a copy stream) alone and while the compute stream replays the
    benchmark's step graph: H2D GB/s into the pool and the share of the loads'
    time hidden under compute."""
    import torch
    g = torch.Generator()
    g.manual_seed(99)
    host = {}
    for k in range(n_adapters):
        at = (torch.randn((rank, d_in), generator=g) / math.sqrt(d_in)).to(torch.bfloat16).view(torch.int16)
        b = (torch.randn((rank, d_out), generator=g) / math.sqrt(rank)).to(torch.bfloat16).view(torch.int16)
        host[k] = (at.pin_memory(), b.pin_memory(), 2.0 * rank)
    target = H.AdapterLayer(d_in, d_out, n_adapters, n_adapters * 4, n_adapters * 4, 16, device=dev)
    pf = H.AdapterPrefetcher(target, host)
    nbytes = sum(a.numel() * 2 + b.numel() * 2 for a, b, _ in host.values())

    def load_all():
        t = pf.prefetch(list(range(n_adapters)))
        pf.end(t, pf.copy)
        for k in range(n_adapters):              # the next round misses again
            s = pf.slots.lookup(k)
            target.evict(s, stream=pf.copy)
            pf.slots.invalidate(s)

    def compute():
        with torch.cuda.stream(stream):
            graph.replay()

    def timed(fn):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pf.copy.wait_event(e0)
        fn()
        stream.wait_stream(pf.copy)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    load_all()
    compute()
    t_l = min(timed(load_all) for _ in range(3))
    t_c = min(timed(compute) for _ in range(3))
    t_b = min(timed(lambda: (load_all(), compute())) for _ in range(3))
    del target, pf
    torch.cuda.empty_cache()
    return {"adapters": n_adapters, "bytes": nbytes, "h2d_gbs": nbytes / (t_l * 1e-3) / 1e9,
            "load_ms": t_l, "compute_ms": t_c, "both_ms": t_b,
            "hidden": (t_l + t_c - t_b) / min(t_l, t_c),
            "what": f"{n_adapters} rank-{rank} adapters ({d_in} -> {d_out}) from pinned host memory into the pool "
                    f"on a copy stream, alone and during one replay of the step graph"}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import heterogeneous_adapter_batching_b200 as H
    from heterogeneous_adapter_batching_b200 import build as lib_build

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if rank == 0:
        lib_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
        dist.barrier()
    H.load_library()

    wl, desc = workload_spec(args.workload)
    P = max(1, args.projections)
    n_layers = ring_layers(wl, args.layers)
    n_layers = (n_layers + P - 1) // P * P
    ring = Ring(wl, n_layers, seed=1234 + rank, device=dev)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    # one step = the plan of the batch + every layer's compute, captured once
    step = ring.step if P == 1 else (lambda s: ring.step_groups(P, s))
    graph, launches_per_step = _capture(step, stream)
    graph.replay()
    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    ev0.record(cur)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(cur)
    torch.cuda.synchronize()
    elapsed_ms = ev0.elapsed_time(ev1)
    # the dominant kernels alone: one layer's compute launches (plan excluded)
    kt = kernel_times(ring, stream, max(10, args.steps), H, P)
    clk = clocks.stop()
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = float(t.item())
        dist.barrier()

    T = wl.T
    tokens_per_step = T * n_layers
    value = tokens_per_step * world * args.steps / (elapsed_ms / 1000.0)
    ms_per_step = elapsed_ms / args.steps

    peak, peak_tf, peak_kind = measured_peaks()
    per_launch_us = kt["kernel_us"] * P
    alg = algorithmic_bytes(wl) * P
    achieved = alg / (per_launch_us * 1e-6) / 1e9
    kname = "compute launches of one layer (plan excluded)"
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": profiled_traffic(args.workload), "peak_source": peak_kind, "kernel": kname,
            "kernel_us": per_launch_us, "algorithmic_bytes_per_launch": alg,
            "launches_per_layer": kt["launches_per_layer"], "plan_us": kt["plan_us"],
            "lora_apply_us": kt["lora_apply_us"],
            "plan": {"gather_jobs": kt["gather_jobs"], "tensor_tiles": kt["tensor_tiles"]}}

    # end to end through the C ABI with host buffers (one layer per step)
    e2e = None
    if not args.no_e2e:
        lay = ring.layers[0]
        Xh = ring.X[0].cpu().pin_memory()
        Yh = ring.Y[0].cpu().pin_memory()
        Ih = ring.ids.cpu().pin_memory()
        Yout = torch.empty_like(Yh).pin_memory()
        Xd, Yd, Id = torch.empty_like(ring.X[0]), torch.empty_like(ring.Y[0]), torch.empty_like(ring.ids)
        with torch.cuda.stream(stream):
            def e2e_step():
                Xd.copy_(Xh, non_blocking=True)
                Yd.copy_(Yh, non_blocking=True)
                Id.copy_(Ih, non_blocking=True)
                lay.apply(Xd, Yd, Id, stream=stream)
                Yout.copy_(Yd, non_blocking=True)
            for _ in range(5):
                e2e_step()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k_e2e = max(20, args.steps)
            e0.record(stream)
            for _ in range(k_e2e):
                e2e_step()
            e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / k_e2e
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        h2d = Xh.numel() * 2 + Yh.numel() * 4 + Ih.numel() * 4
        e2e = {"value": T * world / (e2e_ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(Yout.numel() * 4), "ms_per_step": e2e_ms,
               "path": "pinned H2D of X, Y_base, ids -> lora_apply (plan + compute kernels) -> D2H of Y, one layer"}

    prefetch = None
    if world == 1 and not args.no_prefetch:
        prefetch = measure_prefetch(dev, H, graph, stream)
    del graph
    ring_footprint = ring.footprint()
    del ring
    torch.cuda.empty_cache()

    per_config = None
    if not args.no_per_config and world == 1:
        per_config = {}
        for name in [n for n in args.per_config.split(",") if n]:
            per_config[name] = measure_config(name, dev, stream, H, max(10, args.steps), peak, peak_tf)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, threads, sample = time_oracle(wl, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(wl, desc, args.layers),
            "gpu_launches": int(launches_per_step * args.steps),
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clk,
            "step": {"layers_per_step": n_layers, "plans_per_step": 1, "cuda_graph": True,
                     "ring_bytes": ring_footprint, "parallelism": f"replicas x{world} (no collective)",
                     "projections_per_launch": P},
            "per_config": per_config,
            "prefetch": prefetch,
        }
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
