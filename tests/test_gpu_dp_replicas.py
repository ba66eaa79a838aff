"""GPU: data-parallel replicas of the library, and the gather-path rule.

Tokens are independent (page "Multi-LoRA Serving Architecture ... (2026)",
"Trade-offs, Gotchas, and What Goes Wrong": each token sees only its own
adapter), so the path shards by tokens with no collective.  Here every shard
of a batch runs through its own library instance (its own pools, slot tables
and workspace, as a replica on another GPU would), one after another on one
GPU; concatenated, the shards must equal the unsharded call bit for bit on
batches without long runs (a shard boundary may cut a long run and move its
tokens from the tile path to the gather path, which rounds differently), and
the oracle.
"""
import numpy as np
import pytest

import workloads as W
from tests import _util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    return H


def _apply(wl, X, Y, ids):
    import torch
    layer = U.make_layer(wl)
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    assert int(layer.err.item()) == 0
    return Y.cpu().numpy()


@pytest.mark.parametrize("name", ["decode_q_proj_7b", "mixed_mlp_up"])
@pytest.mark.parametrize("world", [2, 3, 4])
def test_replicas_reassemble_the_unsharded_batch(H, name, world):
    wl = W.by_name(name)
    X, Y, ids = U.dev_inputs(wl)
    full = _apply(wl, X, Y.clone(), ids)
    parts = []
    for rank in range(world):
        lo, hi = W.shard_tokens(wl.T, rank, world)
        parts.append(_apply(wl, X[lo:hi].contiguous(), Y[lo:hi].clone(), ids[lo:hi].contiguous()))
    assert np.array_equal(np.concatenate(parts), full)
    ref, _ = U.oracle_full(wl)
    U.assert_parity(full, ref, wl.Y_base)


@pytest.mark.parametrize("S,T,split", [(300, 64, True), (300, 63, False), (255, 200, False), (32, 64, False)])
def test_gather_path_rule(H, S, T, split):
    """LORA_GATHER_AUTO takes the split pair (plan + shrink + expand) for one
    projection over a pool of >= 256 slots with >= 64 tokens, the cluster kernel
    (plan + one launch) otherwise; both give the same bits."""
    import torch
    old = {k: H.lora_get_option(k) for k in (H.OPT_GATHER_PATH, H.OPT_LONG_SEGMENT)}
    H.lora_set_option(H.OPT_LONG_SEGMENT, 0)     # no tile launches: count the gather launches alone
    try:
        wl = W.random_small(seed=S + T, T=T, d_in=256, d_out=512, S=S, ranks=(4, 16, 64), p_none=0.1)
        X, Y, ids = U.dev_inputs(wl)
        layer = U.make_layer(wl)
        H.lora_set_option(H.OPT_GATHER_PATH, H.GATHER_AUTO)
        Ya = Y.clone()
        layer.apply(X, Ya, ids)
        n_auto = H.lora_last_launch_count()
        H.lora_set_option(H.OPT_GATHER_PATH, H.GATHER_CLUSTER if split else H.GATHER_SPLIT)
        Yo = Y.clone()
        layer.apply(X, Yo, ids)
        torch.cuda.synchronize()
        assert n_auto == (3 if split else 2)
        assert torch.equal(Ya, Yo)
        ref, _ = U.oracle_full(wl)
        U.assert_parity(Ya.cpu().numpy(), ref, wl.Y_base)
    finally:
        for k, v in old.items():
            H.lora_set_option(k, v)
