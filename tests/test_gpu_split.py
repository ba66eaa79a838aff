"""GPU: the split gather path (a shrink kernel writing per-quarter partials of v,
then an expand kernel) against the cluster gather kernel and the fp64 oracle.

Both gather paths take the same arithmetic steps in the same order (d_in in the
same quarters, each warp's 16-column steps, warp-order and quarter-order sums,
pages then high/low parts of v in the expand), so Y must agree bit for bit;
each is also checked against the oracle within |err| <= 2e-3 + 1e-2 |ref|.
Page "Multi-LoRA Serving in Production", section "Segmented Gather
Matrix-Vector Multiplication (SGMV)": shrink, then scaled expand.
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


@pytest.fixture(autouse=True)
def _restore_options(H):
    keys = (H.OPT_LONG_SEGMENT, H.OPT_DECODE_JOB_TOKENS, H.OPT_GATHER_PATH)
    old = {k: H.lora_get_option(k) for k in keys}
    yield
    for k, v in old.items():
        H.lora_set_option(k, v)


def _apply(H, wl, path, layer=None):
    import torch
    H.lora_set_option(H.OPT_GATHER_PATH, path)
    layer = layer or U.make_layer(wl)
    X, Y, ids = U.dev_inputs(wl)
    layer.err.zero_()
    layer.apply(X, Y, ids)
    n_launch = H.lora_last_launch_count()
    torch.cuda.synchronize()
    return Y.cpu().numpy(), int(layer.err.item()), n_launch, layer


def _both(H, wl, delta_rel=U.DELTA_REL_GATHER):
    Ys, es, ns, layer = _apply(H, wl, H.GATHER_SPLIT)
    Yc, ec, nc, _ = _apply(H, wl, H.GATHER_CLUSTER, layer)
    assert es == ec
    assert np.array_equal(Ys, Yc)
    ref, rerr = U.oracle_full(wl)
    assert es == rerr
    U.assert_parity(Ys, ref, wl.Y_base, delta_rel=delta_rel)
    return ns, nc


@pytest.mark.parametrize("job_tokens", [1, 3, 16])
@pytest.mark.parametrize("seed,T,d_in,d_out,S", [
    (1, 1, 64, 64, 3), (2, 7, 24, 40, 5), (3, 33, 264, 136, 9), (4, 100, 512, 1032, 17),
    (5, 257, 8, 8, 4), (6, 64, 1000, 2000, 40), (7, 300, 1032, 4104, 150),
])
def test_split_equals_cluster_random(H, seed, T, d_in, d_out, S, job_tokens):
    """Ragged widths (not multiples of 16 or 64), ranks 1..64 that are not multiples
    of 16, id = -1 tokens, jobs of 1..16 tokens, and (S = 150) slot tables read
    from global memory."""
    H.lora_set_option(H.OPT_DECODE_JOB_TOKENS, job_tokens)
    wl = W.random_small(seed=seed, T=T, d_in=d_in, d_out=d_out, S=S, ranks=(1, 4, 8, 15, 16, 17, 33, 64),
                        p_none=0.15)
    ns, nc = _both(H, wl)
    # one projection's long runs: a tile shrink launch and a tile expand launch
    tiles = 2 if T >= H.lora_get_option(H.OPT_LONG_SEGMENT) else 0
    assert ns == 3 + tiles and nc == 2 + tiles      # plan + shrink + expand | plan + cluster kernel (+ tile launches)


@pytest.mark.parametrize("name", ["decode_q_proj_7b", "mixed_mlp_up", "mixed_mlp_down"])
def test_split_equals_cluster_configs(H, name):
    wl = W.by_name(name)
    _both(H, wl)


@pytest.mark.parametrize("regime,T", [("one", 1), ("one", 64), ("distinct", 64), ("distinct", 1024)])
def test_split_equals_cluster_sweep(H, regime, T):
    wl = W.sweep_8b(T=T, regime=regime)
    _both(H, wl, delta_rel=U.DELTA_REL_TENSOR)


def test_split_with_long_runs(H):
    """Short segments on the split path next to long runs on the tensor-core tiles."""
    H.lora_set_option(H.OPT_LONG_SEGMENT, 16)
    wl = W.segments(6, [40, 200, 3, 130, 60, 9, 300], 512, 768, S=5, reuse=True)
    _both(H, wl, delta_rel=U.DELTA_REL_TENSOR)


def test_split_multi_projection_matches_single_calls(H):
    """lora_apply_multi on the split path (a shrink + expand pair per projection)
    equals the cluster kernel's one launch over all projections, bit for bit."""
    import dataclasses
    import torch
    base = W.random_small(seed=12, T=64, d_in=4096, d_out=4096, S=32, ranks=(4, 16, 64), p_none=0.1)
    wls = [base] + [dataclasses.replace(W._finish(f"p{i}", 500 + i, 4096, d, base.ids, base.ranks()), X=base.X)
                    for i, d in enumerate([1024, 1024])]
    layers = [U.make_layer(w) for w in wls]
    X, _, ids = U.dev_inputs(base)
    out = {}
    for path in (H.GATHER_SPLIT, H.GATHER_CLUSTER):
        H.lora_set_option(H.OPT_GATHER_PATH, path)
        Ys = [U.dev_inputs(w)[1] for w in wls]
        H.apply_multi(layers, X, Ys, ids)
        torch.cuda.synchronize()
        out[path] = [Y.cpu().numpy() for Y in Ys]
    for w, a, b in zip(wls, out[H.GATHER_SPLIT], out[H.GATHER_CLUSTER]):
        assert np.array_equal(a, b), w.name
        ref, _ = U.oracle_full(w)
        U.assert_parity(a, ref, w.Y_base)


def test_split_planned_over_many_layers(H):
    """One plan applied to several layers in a row on one stream (the expand of a
    layer and the shrink of the next overlap through programmatic launches):
    every layer matches its own single call."""
    import torch
    H.lora_set_option(H.OPT_GATHER_PATH, H.GATHER_SPLIT)
    base = W.decode_q_proj_7b()
    wls = [W._finish(f"l{i}", 700 + i, 4096, 4096, base.ids, base.ranks()) for i in range(4)]
    layers = [U.make_layer(w) for w in wls]
    ws = layers[0].ws
    X = [U.dev_inputs(w)[0] for w in wls]
    Y = [U.dev_inputs(w)[1] for w in wls]
    ids = U.dev_inputs(base)[2]
    layers[0].plan(ids, ws=ws)
    for lay, x, y in zip(layers, X, Y):
        lay.apply_planned(x, y, ws=ws)
    torch.cuda.synchronize()
    for w, y in zip(wls, Y):
        ref, _ = U.oracle_full(w)
        U.assert_parity(y.cpu().numpy(), ref, w.Y_base)


def test_split_bad_page_and_empty_slot(H):
    """A page outside the pool and an evicted slot on the split path: their rows
    stay Y_base, the error bits are set, every other row equals the clean run."""
    import torch
    H.lora_set_option(H.OPT_GATHER_PATH, H.GATHER_SPLIT)
    wl = W.random_small(seed=74, T=80, d_in=256, d_out=200, S=6, ranks=(16, 33, 64), p_none=0.0)
    Yc, err, _, layer = _apply(H, wl, H.GATHER_SPLIT)
    assert err == 0
    bad, gone = int(wl.ids[5]), int(wl.ids[40])
    if gone == bad:
        gone = int(next(i for i in wl.ids if i != bad))
    layer.page_table[bad, 1, 0] = H.lora_pool_num_pages(layer.pool_b) + 1
    layer.evict(gone)
    X, Y, ids = U.dev_inputs(wl)
    layer.err.zero_()
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    Yb = Y.cpu().numpy()
    assert int(layer.err.item()) == H.DEV_ERR_BAD_PAGE | H.DEV_ERR_EMPTY_SLOT
    rows = (wl.ids == bad) | (wl.ids == gone)
    assert np.array_equal(Yb[rows], wl.Y_base[rows])
    assert np.array_equal(Yb[~rows], Yc[~rows])
