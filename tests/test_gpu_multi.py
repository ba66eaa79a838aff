"""GPU parity of lora_apply_multi: several projections that read the same X
in one call (page "Multi-LoRA Serving Architecture ... (2026)", section "The
memory arithmetic that makes it work": an all-linear adapter has its own A and
B for each projection of a layer, with per-projection output widths).

Each projection is checked against the fp64 oracle and bit-exactly against a
separate lora_apply on that projection alone.
"""
import dataclasses

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
    old = {k: H.lora_get_option(k) for k in (H.OPT_LONG_SEGMENT, H.OPT_DECODE_JOB_TOKENS, H.OPT_GATHER_PATH)}
    yield
    for k, v in old.items():
        H.lora_set_option(k, v)


def _projections(base, d_outs, seed, empty=()):
    """base's X, ids and slot ranks with fresh adapters (own seed) for every
    further output width; slots in `empty` hold no adapter in projection 1."""
    wls = [base]
    for i, d in enumerate(d_outs):
        ranks = base.ranks()
        if i == 0:
            for k in empty:
                ranks[k] = 0
        w = W._finish(f"{base.name}_p{i + 1}", seed * 1000 + i + 1, base.d_in, d, base.ids, ranks)
        wls.append(dataclasses.replace(w, X=base.X))
    return wls


def _run(H, wls):
    import torch
    layers = [U.make_layer(w) for w in wls]
    X, _, ids = U.dev_inputs(wls[0])
    Ys = [U.dev_inputs(w)[1] for w in wls]
    layers[0].err.zero_()
    H.apply_multi(layers, X, Ys, ids)
    _run.launches = H.lora_last_launch_count()
    torch.cuda.synchronize()
    multi = [Y.cpu().numpy() for Y in Ys]
    err = int(layers[0].err.item())
    single = []
    for lay, w in zip(layers, wls):
        _, Y, _ = U.dev_inputs(w)
        lay.err.zero_()
        lay.apply(X, Y, ids)
        torch.cuda.synchronize()
        single.append(Y.cpu().numpy())
    return multi, single, err


@pytest.mark.parametrize("seed,T,d_in,d_outs,S", [
    (11, 7, 256, [256, 64, 520], 5),
    (12, 64, 4096, [4096, 1024, 1024], 32),
    (13, 200, 384, [136, 1032], 17),
    (14, 1, 64, [64, 64, 64, 64, 64, 64, 64], 3),
])
def test_multi_matches_single_and_oracle(H, seed, T, d_in, d_outs, S):
    base = W.random_small(seed=seed, T=T, d_in=d_in, d_out=d_outs[0], S=S, ranks=(1, 4, 8, 15, 16, 17, 33, 64),
                          p_none=0.1)
    wls = _projections(base, d_outs[1:], seed)
    multi, single, err = _run(H, wls)
    assert err == 0
    for w, m, s in zip(wls, multi, single):
        assert np.array_equal(m, s), w.name
        ref, rerr = U.oracle_full(w)
        assert rerr == 0
        U.assert_parity(m, ref, w.Y_base)


def test_multi_long_runs(H):
    """Long runs of all projections take one tile launch; short segments the shared
    gather launch (cluster path: plan + gather + tiles = 3 launches)."""
    H.lora_set_option(H.OPT_LONG_SEGMENT, 16)
    H.lora_set_option(H.OPT_GATHER_PATH, H.GATHER_CLUSTER)
    base = W.segments(21, [5, 40, 300, 2, 129], 256, 512, 8, reuse=True)
    wls = _projections(base, [256, 1032], 21)
    multi, single, err = _run(H, wls)
    assert _run.launches == 3
    assert err == 0
    for w, m, s in zip(wls, multi, single):
        assert np.array_equal(m, s), w.name
        ref, _ = U.oracle_full(w)
        U.assert_parity(m, ref, w.Y_base, delta_rel=U.DELTA_REL_TENSOR)


def test_multi_slot_empty_in_one_projection(H):
    """A slot empty in projection 1 (rank 0) leaves that projection's rows of its
    tokens unchanged; projection 0 still applies it and no error bit is set."""
    base = W.random_small(seed=31, T=40, d_in=128, d_out=128, S=6, ranks=(4, 16, 64), p_none=0.0)
    wls = _projections(base, [192], 31, empty=(2,))
    multi, single, err = _run(H, wls)
    assert err == 0
    assert np.array_equal(multi[1], single[1])
    rows = base.ids == 2
    assert rows.any()
    assert np.array_equal(multi[1][rows], wls[1].Y_base[rows])
    for w, m in zip(wls, multi):
        ref, _ = U.oracle_full(w)
        U.assert_parity(m, ref, w.Y_base)


def test_multi_rejects_bad_arguments(H):
    import torch
    base = W.random_small(seed=41, T=4, d_in=64, d_out=64, S=3)
    wls = _projections(base, [64], 41)
    layers = [U.make_layer(w) for w in wls]
    X, Y, ids = U.dev_inputs(base)
    with pytest.raises(H.LoraError):   # 9 projections
        H.apply_multi(layers * 5, X, [Y] * 10, ids)
    other = U.make_layer(W.random_small(seed=42, T=4, d_in=128, d_out=64, S=3))
    with pytest.raises(H.LoraError):   # width mismatch in projection 1
        H.apply_multi([layers[0], other], X, [Y, Y.clone()], ids)
    torch.cuda.synchronize()


def test_multi_planned_matches_multi(H):
    """The planned variant over the plan of lora_plan equals the one-call form."""
    import torch
    base = W.random_small(seed=51, T=96, d_in=512, d_out=512, S=12, ranks=(4, 8, 16, 64), p_none=0.1)
    wls = _projections(base, [1024, 256], 51)
    layers = [U.make_layer(w) for w in wls]
    X, _, ids = U.dev_inputs(base)
    Ya = [U.dev_inputs(w)[1] for w in wls]
    Yb = [U.dev_inputs(w)[1] for w in wls]
    H.apply_multi(layers, X, Ya, ids)
    layers[0].plan(ids)
    H.apply_multi(layers, X, Yb, None)
    torch.cuda.synchronize()
    for a, b in zip(Ya, Yb):
        assert torch.equal(a, b)
