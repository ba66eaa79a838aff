"""Tensor-parallel schedule of the adapter branch on CPU ranks (gloo, world size 2).

Page "Multi-LoRA Serving in Production", sections "Partitioning Rules for
Linear Layers" and "S-LoRA TP Communication Optimization".  Each rank runs
TPLoRA.forward (the real schedule: which shard, which collective, in which
order) with the fp64 oracle standing in for the kernels through the `ops` hook;
the reassembled output must equal the unsharded oracle:

* column-parallel: A replicated, B split by columns, no collective;
* row-parallel: A split by rows, B replicated, one all-reduce of base +
  adapter partials;
* S-LoRA variant: A split by rows, B split by columns, all-reduce of the
  rank-r partial v, then the layer's all-reduce.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W
from heterogeneous_adapter_batching_b200 import tp


def test_shard_range_covers_in_aligned_blocks():
    for n in (8, 64, 4096, 11008, 14336, 1000):
        for world in (1, 2, 3, 4, 8):
            blocks = [tp.shard_range(n, r, world) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == n
            for (a, b), (c, d) in zip(blocks, blocks[1:]):
                assert b == c
            assert all(lo % 8 == 0 and hi % 8 == 0 and hi >= lo for lo, hi in blocks)
            sizes = [hi - lo for lo, hi in blocks]
            assert max(sizes) - min(sizes) <= 8
    with pytest.raises(ValueError):
        tp.shard_range(12, 0, 2)


class HostLayer:
    """Host stand-in for one rank's device state: the shard's A and B per slot."""

    def __init__(self, d_in, d_out, S):
        self.d_in, self.d_out, self.S = d_in, d_out, S
        self.A, self.B = [None] * S, [None] * S
        self.sc = np.zeros(S, np.float32)

    def load(self, slot, rank, alpha, a_t, b, page_ids=None, stream=None):
        self.A[slot] = a_t.numpy().astype(np.float32).T.copy()
        self.B[slot] = b.numpy().astype(np.float32).copy()
        self.sc[slot] = np.float32(alpha) / np.float32(rank)


class HostOps:
    """The oracle in place of the kernels (test only)."""

    @staticmethod
    def apply(layer, X, Y, ids, stream=None):
        from oracle import lora_oracle as O
        out, _ = O.lora_apply(X.numpy(), Y.numpy(), ids.numpy(), layer.A, layer.B, layer.sc)
        Y.copy_(torch.from_numpy(out))

    @staticmethod
    def shrink(layer, X, ids, V, stream=None):
        from oracle import lora_oracle as O
        v, _ = O.lora_shrink(X.numpy(), ids.numpy(), layer.A)
        ok = ~np.isnan(v)
        Vn = V.numpy()
        Vn[ok] = v[ok]

    @staticmethod
    def expand_add_block(layer, V, Y, col0, ids, stream=None):
        from oracle import lora_oracle as O
        blk = Y[:, col0:col0 + layer.d_out]
        out, _ = O.lora_expand_add(V.numpy(), blk.numpy(), ids.numpy(), layer.B, layer.sc)
        blk.copy_(torch.from_numpy(out))


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
        from oracle import lora_oracle as O
        wl = W.random_small(seed=41, T=29, d_in=48, d_out=40, S=5, ranks=(1, 4, 8, 16), p_none=0.2)
        A = [a.A for a in wl.adapters]
        Bm = [a.B for a in wl.adapters]
        sc = wl.scales_f32()
        W0 = np.random.default_rng(42).standard_normal((wl.d_in, wl.d_out))
        X = torch.from_numpy(wl.X.astype(np.float64))
        ids = torch.from_numpy(wl.ids)
        ref, _ = O.lora_apply(wl.X, wl.X.astype(np.float64) @ W0, wl.ids, A, Bm, sc)
        results = {}
        for mode in (tp.COLUMN, tp.ROW, tp.ROW_V_EXCHANGE):
            sh = tp.TPLoRA(mode, wl.d_in, wl.d_out, wl.S, 0, wl.T, rank, world, ops=HostOps,
                           layer=HostLayer(*_shard_dims(mode, wl, rank, world), wl.S))
            for i, a in enumerate(wl.adapters):
                sh.load(i, a.rank, a.alpha, torch.from_numpy(a.A.T.copy()), torch.from_numpy(a.B.copy()))
            X_local = X[:, sh.in_lo:sh.in_hi].contiguous()
            W0_local = W0[sh.in_lo:sh.in_hi, sh.out_lo:sh.out_hi] if mode == tp.COLUMN else W0[sh.in_lo:sh.in_hi]
            Y = torch.from_numpy(X_local.numpy() @ W0_local)      # this rank's base output (block or partial)
            sh.forward(X_local, Y, ids)
            if mode == tp.COLUMN:   # uneven blocks (40 columns = 24 + 16): gather padded, then trim
                spans = [tp.shard_range(wl.d_out, r, world) for r in range(world)]
                wmax = max(hi - lo for lo, hi in spans)
                pad = torch.zeros((wl.T, wmax), dtype=torch.float64)
                pad[:, :Y.shape[1]] = Y
                blocks = [torch.zeros_like(pad) for _ in range(world)]
                dist.all_gather(blocks, pad)
                Y = torch.cat([b[:, :hi - lo] for b, (lo, hi) in zip(blocks, spans)], dim=1)
            results[mode] = Y.numpy()
        if rank == 0:
            ok = {m: bool(np.allclose(y, ref, rtol=1e-11, atol=1e-11)) for m, y in results.items()}
            q.put(ok)
    finally:
        dist.destroy_process_group()


def _shard_dims(mode, wl, rank, world):
    if mode == tp.COLUMN:
        lo, hi = tp.shard_range(wl.d_out, rank, world)
        return wl.d_in, hi - lo
    ilo, ihi = tp.shard_range(wl.d_in, rank, world)
    if mode == tp.ROW:
        return ihi - ilo, wl.d_out
    olo, ohi = tp.shard_range(wl.d_out, rank, world)
    return ihi - ilo, ohi - olo


def test_tp_schedules_reassemble_the_unsharded_branch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs)
    ok = q.get(timeout=5)
    assert ok == {tp.COLUMN: True, tp.ROW: True, tp.ROW_V_EXCHANGE: True}, ok
