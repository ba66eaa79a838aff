"""Shared helpers of the GPU tests: upload a seeded workload through the C ABI
and compare device results with the fp64 oracle."""
from __future__ import annotations

import numpy as np

import workloads as W

# Required tolerance per element (fp32 accumulate): |err| <= 2e-3 + 1e-2 |ref|.
ATOL, RTOL = 2e-3, 1e-2
# A stricter bound on the adapter delta alone, relative to its largest magnitude.
# It separates a wrong rank row / adapter / scale (O(1) relative) from rounding.
DELTA_REL_GATHER = 1e-4     # fp32 accumulation; v enters the expand as two bf16 parts (~16 bits)
DELTA_REL_TENSOR = 2e-4     # the same on the tensor-core tiles (tcgen05, fp32 accumulation, v in two parts)


def make_layer(wl: W.Workload, max_tokens=None, shared_pool=False, extra_pages=0):
    import torch
    from heterogeneous_adapter_batching_b200 import AdapterLayer
    layer = AdapterLayer(wl.d_in, wl.d_out, wl.S, wl.pages_a + extra_pages, wl.pages_b + extra_pages,
                         max(1, max_tokens if max_tokens is not None else wl.T), shared_pool=shared_pool)
    for i in range(wl.S):
        a = wl.adapters[i]
        if a is None:
            continue
        at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16)).cuda()
        b = torch.from_numpy(W.bf16_bits(a.B).view(np.int16)).cuda()
        pid = None if shared_pool else torch.from_numpy(np.ascontiguousarray(wl.page_ids[i]))
        layer.load(i, a.rank, a.alpha, at, b, page_ids=pid)
    return layer


def dev_inputs(wl: W.Workload):
    import torch
    X = torch.from_numpy(W.bf16_bits(wl.X).view(np.int16)).cuda().view(torch.bfloat16)
    Y = torch.from_numpy(wl.Y_base.copy()).cuda()
    ids = torch.from_numpy(wl.ids.copy()).cuda()
    return X, Y, ids


def oracle_full(wl: W.Workload, nthreads=0):
    from oracle import build_oracle as OC
    A = [None if a is None else a.A for a in wl.adapters]
    B = [None if a is None else a.B for a in wl.adapters]
    return OC.lora_apply_c(wl.X, wl.Y_base, wl.ids, A, B, wl.scales_f32(), nthreads=nthreads)


def assert_parity(Y_dev: np.ndarray, Y_ref: np.ndarray, Y_base: np.ndarray, delta_rel=DELTA_REL_GATHER):
    Y_dev = np.asarray(Y_dev, np.float64)
    err = np.abs(Y_dev - Y_ref)
    bound = ATOL + RTOL * np.abs(Y_ref)
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} elements outside 2e-3+1e-2|ref|; worst {err.max():.3e}"
    d_ref = Y_ref - np.asarray(Y_base, np.float64)
    d_dev = Y_dev - np.asarray(Y_base, np.float64)
    scale = np.abs(d_ref).max()
    if scale > 0:
        worst = np.abs(d_dev - d_ref).max()
        assert worst <= delta_rel * scale, f"delta error {worst:.3e} > {delta_rel:g} * {scale:.3e}"


def expected_work(ids, ranks, long_thresh: int, job_tokens: int):
    """(n_jobs, n_tiles) the plan should produce: maximal runs of one valid slot with at
    least long_thresh tokens become ceil(len/128) tiles; the other valid tokens of
    each slot are split into ceil(count/job_tokens) gather jobs."""
    ids = np.asarray(ids)
    S = len(ranks)
    valid = np.array([(0 <= i < S) and ranks[i] > 0 for i in ids], dtype=bool)
    T = len(ids)
    in_long = np.zeros(T, dtype=bool)
    n_tiles = 0
    if long_thresh > 0 and T >= long_thresh:
        t = 0
        while t < T:
            if not valid[t]:
                t += 1
                continue
            e = t
            while e + 1 < T and valid[e + 1] and ids[e + 1] == ids[t]:
                e += 1
            L = e - t + 1
            if L >= long_thresh:
                in_long[t:e + 1] = True
                n_tiles += (L + 127) // 128
            t = e + 1
    n_jobs = 0
    short = ids[valid & ~in_long]
    for k, c in zip(*np.unique(short, return_counts=True)):
        n_jobs += (int(c) + job_tokens - 1) // job_tokens
    return n_jobs, n_tiles


def job_size_candidates(jmax: int):
    """Job sizes the plan chooses from under the cap jmax."""
    return sorted({min(4, jmax), min(8, jmax), jmax})


def plan_job_tokens(ws):
    """Job size the plan chose (PlanHeader field 6 at the head of the workspace)."""
    return int(ws[:32].cpu().numpy().view(np.int32)[6])


def plan_counts(ws):
    """(n_valid, n_seg, n_jobs, n_tiles) from the head of a workspace the library
    filled (the plan header is the workspace's first 16 bytes)."""
    h = ws[:16].cpu().numpy().view(np.int32)
    return tuple(int(x) for x in h[:4])
