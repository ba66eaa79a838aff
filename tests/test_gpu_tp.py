"""GPU: tensor-parallel shards of the adapter branch through the library.

Page "Multi-LoRA Serving in Production", sections "Partitioning Rules for
Linear Layers" and "S-LoRA TP Communication Optimization".  One device runs
every rank's library calls in turn; device-side sums and concatenations stand
in for the collectives (the real schedule with gloo collectives is checked in
test_tp_sharding.py).  Column-parallel shards reassemble the unsharded
lora_apply bit for bit (the same shrink, the same per-column expand); the
row-parallel sum and the S-LoRA v exchange match the fp64 oracle within the
tolerance.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import workloads as W
from tests import _util as U

pytestmark = pytest.mark.gpu


def _shards(tp, mode, wl, world):
    import torch
    sh = []
    for r in range(world):
        t = tp.TPLoRA(mode, wl.d_in, wl.d_out, wl.S, wl.pages_a + wl.pages_b, wl.T, r, world)
        for i, a in enumerate(wl.adapters):
            if a is None:
                continue
            at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16)).cuda()
            b = torch.from_numpy(W.bf16_bits(a.B).view(np.int16)).cuda()
            t.load(i, a.rank, a.alpha, at, b)
        sh.append(t)
    return sh


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("seed,T,d_in,d_out,S", [(1, 64, 4096, 4096, 32), (2, 37, 512, 1032, 9)])
def test_column_parallel_is_bit_exact(seed, T, d_in, d_out, S, world):
    import torch
    from heterogeneous_adapter_batching_b200 import tp
    wl = W.random_small(seed=seed, T=T, d_in=d_in, d_out=d_out, S=S, ranks=(4, 8, 16, 33, 64), p_none=0.1)
    full = U.make_layer(wl)
    X, Y, ids = U.dev_inputs(wl)
    full.apply(X, Y, ids)
    blocks = []
    for sh in _shards(tp, tp.COLUMN, wl, world):
        Yk = U.dev_inputs(wl)[1][:, sh.out_lo:sh.out_hi].contiguous()
        sh.local_apply(X, Yk, ids)
        blocks.append(Yk)
    torch.cuda.synchronize()
    got = torch.cat(blocks, dim=1).cpu().numpy()
    assert np.array_equal(got, Y.cpu().numpy())
    ref, _ = U.oracle_full(wl)
    U.assert_parity(got, ref, wl.Y_base)


@pytest.mark.parametrize("mode", ["row", "row_v_exchange"])
@pytest.mark.parametrize("world", [2, 4])
def test_row_parallel_sum_matches_oracle(mode, world):
    import torch
    from heterogeneous_adapter_batching_b200 import tp
    wl = W.random_small(seed=3, T=70, d_in=4096, d_out=1024, S=12, ranks=(4, 8, 16), p_none=0.1)
    X, Y0, ids = U.dev_inputs(wl)
    shards = _shards(tp, mode, wl, world)
    partials = []
    for k, sh in enumerate(shards):
        Xk = X[:, sh.in_lo:sh.in_hi].contiguous()
        Yk = Y0.clone() if k == 0 else torch.zeros_like(Y0)      # the base partials sum to Y_base
        partials.append((sh, Xk, Yk))
    if mode == tp.ROW:
        for sh, Xk, Yk in partials:
            sh.local_apply(Xk, Yk, ids)
    else:
        Vs = []
        for sh, Xk, _ in partials:
            V = torch.zeros((wl.T, 64), dtype=torch.float32, device="cuda")
            sh.local_shrink(Xk, ids, V)
            Vs.append(V)
        V_sum = torch.stack(Vs).sum(0)                          # the all-reduce of v
        for sh, _, Yk in partials:
            sh.local_expand(V_sum, Yk, ids)
    Y = torch.stack([p[2] for p in partials]).sum(0)            # the layer's all-reduce
    torch.cuda.synchronize()
    ref, _ = U.oracle_full(wl)
    U.assert_parity(Y.cpu().numpy(), ref, wl.Y_base, delta_rel=1e-3)


_FORWARD = r'''
import os, sys, numpy as np, torch, torch.distributed as dist
sys.path.insert(0, os.environ["ROOT"])
import workloads as W
from tests import _util as U
from heterogeneous_adapter_batching_b200 import tp
torch.cuda.set_device(0)
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%s" % os.environ["PORT"], rank=0, world_size=1)
wl = W.random_small(seed=5, T=33, d_in=256, d_out=320, S=6, ranks=(4, 16), p_none=0.1)
ref, _ = U.oracle_full(wl)
ok = True
for mode in (tp.COLUMN, tp.ROW, tp.ROW_V_EXCHANGE):
    sh = tp.TPLoRA(mode, wl.d_in, wl.d_out, wl.S, wl.pages_a + wl.pages_b, wl.T, 0, 1)
    for i, a in enumerate(wl.adapters):
        at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16)).cuda()
        b = torch.from_numpy(W.bf16_bits(a.B).view(np.int16)).cuda()
        sh.load(i, a.rank, a.alpha, at, b)
    X, Y, ids = U.dev_inputs(wl)
    sh.forward(X, Y, ids)
    torch.cuda.synchronize()
    U.assert_parity(Y.cpu().numpy(), ref, wl.Y_base)
dist.destroy_process_group()
print("forward ok")
'''


def test_forward_with_nccl_group_of_one():
    """TPLoRA.forward with a real NCCL process group (one rank: every collective is
    an identity), so the library calls and the NCCL calls run in one schedule."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, ROOT=root, PORT=str(port))
    out = subprocess.run([sys.executable, "-c", _FORWARD], capture_output=True, text=True, timeout=300, env=env,
                         cwd=root)
    assert out.returncode == 0, out.stderr[-3000:]
    assert "forward ok" in out.stdout
