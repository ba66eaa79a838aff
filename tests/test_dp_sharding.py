"""Data-parallel replicas on CPU ranks (gloo, world size 2): tokens are
independent, so splitting the batch across ranks and concatenating the
shards' results reproduces the unsharded batch exactly (page
"Multi-LoRA Serving Architecture ... (2026)", "Trade-offs, Gotchas": each
token only sees its own adapter).  The path needs no collective; gloo is
used here only to bring the shards back for the comparison."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import build_oracle as OC
        wl = W.random_small(seed=31, T=37, d_in=40, d_out=24, S=5, ranks=(1, 4, 8), p_none=0.2)
        lo, hi = W.shard_tokens(wl.T, rank, world)
        A = [a.A for a in wl.adapters]
        B = [a.B for a in wl.adapters]
        Y, err = OC.lora_apply_c(wl.X[lo:hi], wl.Y_base[lo:hi], wl.ids[lo:hi], A, B, wl.scales_f32(), nthreads=1)
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([hi - lo]))
        mx = int(max(s.item() for s in sizes))
        pad = torch.zeros((mx, wl.d_out), dtype=torch.float64)
        pad[: hi - lo] = torch.from_numpy(Y)
        outs = [torch.zeros_like(pad) for _ in range(world)]
        dist.all_gather(outs, pad)
        if rank == 0:
            full = np.concatenate([o[: int(s.item())].numpy() for o, s in zip(outs, sizes)])
            ref, _ = OC.lora_apply_c(wl.X, wl.Y_base, wl.ids, A, B, wl.scales_f32(), nthreads=1)
            q.put(bool(np.array_equal(full, ref)) and full.shape == ref.shape)
    finally:
        dist.destroy_process_group()


def test_shard_tokens_partition():
    for T in (0, 1, 5, 64, 1023):
        for world in (1, 2, 3, 8):
            rngs = [W.shard_tokens(T, r, world) for r in range(world)]
            assert rngs[0][0] == 0 and rngs[-1][1] == T
            for a, b in zip(rngs, rngs[1:]):
                assert a[1] == b[0]
            sizes = [h - l for l, h in rngs]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_shards_reassemble_exactly():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=5) is True
