"""GPU parity: liblora (through the C ABI) against the fp64 oracle, element by element.

Tolerance per element (fp32 accumulate): |err| <= 2e-3 + 1e-2 |ref|, plus a
stricter bound on the adapter delta (see tests/_util.py).  All indexing
(plan, pages, which rows change) is checked bit-exactly.
"""
import numpy as np
import pytest

import workloads as W
from tests import _util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import torch
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    torch.cuda.init()
    return H


@pytest.fixture(autouse=True)
def _restore_options(H):
    old = {k: H.lora_get_option(k) for k in (H.OPT_LONG_SEGMENT, H.OPT_DECODE_JOB_TOKENS)}
    yield
    for k, v in old.items():
        H.lora_set_option(k, v)


def _run_apply(H, wl, **kw):
    import torch
    layer = U.make_layer(wl, **kw)
    X, Y, ids = U.dev_inputs(wl)
    layer.err.zero_()
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    return Y.cpu().numpy(), int(layer.err.item()), layer


def test_tiny_config(H):
    wl = W.tiny()
    Y, err, _ = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base)


@pytest.mark.parametrize("job_tokens", [1, 3, 4, 9, 16])
@pytest.mark.parametrize("seed,T,d_in,d_out,S", [
    (1, 1, 64, 64, 3), (2, 7, 24, 40, 5), (3, 33, 264, 136, 9), (4, 100, 512, 1032, 17),
    (5, 257, 8, 8, 4), (6, 64, 1000, 2000, 40),
])
def test_random_small(H, seed, T, d_in, d_out, S, job_tokens):
    H.lora_set_option(H.OPT_DECODE_JOB_TOKENS, job_tokens)
    wl = W.random_small(seed=seed, T=T, d_in=d_in, d_out=d_out, S=S, ranks=(1, 4, 8, 15, 16, 17, 33, 64),
                        p_none=0.15)
    Y, err, _ = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base)


def _check_job_size(layer, wl, expect):
    """The plan's job size and job count.  On a B200 the gather kernel keeps
    about 33 clusters: 64 Zipf decode tokens give 25 jobs of 4 (fewer than
    the clusters, so the size stays 4); 256 MLP tokens give about 100 (so the
    size grows to 16, still leaving more jobs than clusters)."""
    jt = U.plan_job_tokens(layer.ws)
    assert jt == expect
    n_jobs = U.plan_counts(layer.ws)[2]
    assert n_jobs == U.expected_work(wl.ids, wl.ranks(), 0, jt)[0]


def test_decode_q_proj_7b_full(H):
    wl = W.decode_q_proj_7b()
    Y, err, layer = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base)
    _check_job_size(layer, wl, 4)


@pytest.mark.parametrize("which", ["up", "down"])
def test_mixed_mlp_full(H, which):
    wl = W.mixed_mlp(which=which)
    Y, err, layer = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base)
    _check_job_size(layer, wl, 16)


def test_prefill_full(H):
    wl = W.prefill()
    Y, err, _ = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)


@pytest.mark.parametrize("regime", ["one", "distinct"])
@pytest.mark.parametrize("T", [1, 16, 64, 256, 1024])
def test_sweep_8b(H, regime, T):
    wl = W.sweep_8b(T=T, regime=regime)
    Y, err, _ = _run_apply(H, wl)
    assert err == 0
    # every token, every adapter's pages: at T = 1024 the fp64 oracle is about
    # 2.4 GFLOP, a few seconds on the host's cores
    ref, rerr = U.oracle_full(wl)
    assert rerr == 0
    U.assert_parity(Y, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)


# ---------------------------------------------------------------------------
# Invariants the pages fix
# ---------------------------------------------------------------------------

def test_zero_b_leaves_y_bit_exact(H):
    import torch
    wl = W.random_small(seed=11, T=50, d_in=256, d_out=320, S=6, ranks=(4, 16, 64))
    layer = U.make_layer(wl)
    # overwrite every B row with zeros through a reload into the same pages
    for i in range(wl.S):
        a = wl.adapters[i]
        layer.evict(i)
        at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16)).cuda()
        b0 = torch.zeros((a.rank, wl.d_out), dtype=torch.int16, device="cuda")
        layer.load(i, a.rank, a.alpha, at, b0, page_ids=torch.from_numpy(wl.page_ids[i].copy()))
    X, Y, ids = U.dev_inputs(wl)
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    assert np.array_equal(Y.cpu().numpy(), wl.Y_base)


def test_permutation_equivariance_bit_exact(H):
    import torch
    wl = W.decode_q_proj_7b(T=64)
    Y1, _, layer = _run_apply(H, wl)
    P = np.random.default_rng(3).permutation(wl.T)
    X, Y, ids = U.dev_inputs(wl)
    Pt = torch.from_numpy(P).cuda()
    X2, Y2, ids2 = X[Pt].contiguous(), Y[Pt].contiguous(), ids[Pt].contiguous()
    layer.apply(X2, Y2, ids2)
    torch.cuda.synchronize()
    assert np.array_equal(Y2.cpu().numpy(), Y1[P])


def test_none_and_invalid_ids(H):
    import torch
    wl = W.random_small(seed=12, T=40, d_in=128, d_out=96, S=5, ranks=(8, 16), p_none=0.0)
    Yc, _, layer = _run_apply(H, wl)
    X, Y, ids = U.dev_inputs(wl)
    ids_h = wl.ids.copy()
    ids_h[[1, 9]] = -1
    ids_h[[3, 20]] = wl.S          # out of range
    ids_h[[5]] = -7                # out of range
    ids.copy_(torch.from_numpy(ids_h))
    layer.err.zero_()
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    Yn = Y.cpu().numpy()
    assert int(layer.err.item()) == H.DEV_ERR_BAD_ID
    for t in (1, 9, 3, 20, 5):
        assert np.array_equal(Yn[t], wl.Y_base[t])
    others = [t for t in range(wl.T) if t not in (1, 9, 3, 20, 5)]
    assert np.array_equal(Yn[others], Yc[others])


def test_evicted_slot_sets_empty_bit_and_skips(H):
    import torch
    wl = W.random_small(seed=13, T=30, d_in=128, d_out=128, S=4, ranks=(16,), p_none=0.0)
    Yc, _, layer = _run_apply(H, wl)
    layer.evict(2)
    X, Y, ids = U.dev_inputs(wl)
    layer.err.zero_()
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    Yn = Y.cpu().numpy()
    assert int(layer.err.item()) == H.DEV_ERR_EMPTY_SLOT
    on2 = wl.ids == 2
    assert on2.any()
    assert np.array_equal(Yn[on2], wl.Y_base[on2])
    assert np.array_equal(Yn[~on2], Yc[~on2])


def test_all_tokens_one_adapter_matches_dense(H):
    """One adapter for the whole batch equals one dense product (fp64 numpy matmul)."""
    wl = W.sweep_8b(T=64, regime="one", pool=4, d_in=1024, d_out=2048)
    Y, err, _ = _run_apply(H, wl)
    i = int(wl.ids[0])
    a = wl.adapters[i]
    s = np.float64(wl.scales_f32()[i])
    ref = wl.Y_base.astype(np.float64) + s * (wl.X.astype(np.float64) @ a.A.astype(np.float64)) @ a.B.astype(np.float64)
    assert err == 0
    U.assert_parity(Y, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)


def test_empty_batch_and_all_none(H):
    import torch
    wl = W.random_small(seed=14, T=16, d_in=64, d_out=64, S=3, ranks=(8,), p_none=1.0)
    Y, err, _ = _run_apply(H, wl)
    assert err == 0 and np.array_equal(Y, wl.Y_base)
    layer = U.make_layer(wl)
    X0 = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    Y0 = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    ids0 = torch.empty((0,), dtype=torch.int32, device="cuda")
    layer.apply(X0, Y0, ids0)
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# The two-step entry points
# ---------------------------------------------------------------------------

def test_shrink_matches_oracle(H):
    import torch
    from oracle import lora_oracle as O
    wl = W.random_small(seed=15, T=70, d_in=520, d_out=64, S=7, ranks=(1, 8, 16, 40, 64), p_none=0.1)
    layer = U.make_layer(wl)
    X, _, ids = U.dev_inputs(wl)
    V = torch.full((wl.T, 64), float("nan"), dtype=torch.float32, device="cuda")
    layer.shrink(X, ids, V)
    torch.cuda.synchronize()
    Vd = V.cpu().numpy()
    Vr, _ = O.lora_shrink(wl.X, wl.ids, [a.A for a in wl.adapters])
    defined = ~np.isnan(Vr)
    assert np.array_equal(np.isnan(Vd), ~defined)          # untouched entries stay NaN
    err = np.abs(Vd[defined] - Vr[defined])
    assert (err <= U.ATOL + U.RTOL * np.abs(Vr[defined])).all()
    assert err.max() <= 1e-4 * np.abs(Vr[defined]).max()


def test_expand_add_matches_oracle(H):
    import torch
    from oracle import lora_oracle as O
    wl = W.random_small(seed=16, T=70, d_in=64, d_out=1000, S=7, ranks=(1, 8, 16, 40, 64), p_none=0.1)
    layer = U.make_layer(wl)
    _, Y, ids = U.dev_inputs(wl)
    Vh = np.random.default_rng(16).standard_normal((wl.T, 64)).astype(np.float32)
    V = torch.from_numpy(Vh).cuda()
    layer.expand_add(V, Y, ids)
    torch.cuda.synchronize()
    ref, _ = O.lora_expand_add(Vh, wl.Y_base, wl.ids, [a.B for a in wl.adapters], wl.scales_f32())
    U.assert_parity(Y.cpu().numpy(), ref, wl.Y_base)


def test_max_slots(H):
    """LORA_MAX_SLOTS = 4096 resident slots: the plan's smallest per-warp table
    and slot tables read from global memory (too many to stage)."""
    wl = W.random_small(seed=61, T=300, d_in=64, d_out=72, S=4096, ranks=(1, 4, 16, 64), p_none=0.05)
    Y, err, _ = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base)


def test_many_tokens(H):
    """32768 decode-style tokens over 64 slots: tens of thousands of gather jobs
    over the persistent clusters (no long runs at this id mix)."""
    wl = W.random_small(seed=62, T=32768, d_in=128, d_out=136, S=64, ranks=(4, 8, 16, 33, 64), p_none=0.1)
    Y, err, layer = _run_apply(H, wl)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base)
    jt = U.plan_job_tokens(layer.ws)
    assert U.plan_counts(layer.ws)[2] == U.expected_work(wl.ids, wl.ranks(), H.lora_get_option(H.OPT_LONG_SEGMENT), jt)[0]


# ---------------------------------------------------------------------------
# Slot tables that name memory outside the pool (LORA_DEV_ERR_BAD_PAGE)
# ---------------------------------------------------------------------------

def _corrupt_and_apply(H, wl, corrupt, thresh=None):
    """Run lora_apply on a clean layer, then again after `corrupt(layer)` edits the
    device slot tables; returns (clean Y, corrupted Y, error word)."""
    import torch
    if thresh is not None:
        H.lora_set_option(H.OPT_LONG_SEGMENT, thresh)
    Yc, err, layer = _run_apply(H, wl)
    assert err == 0
    corrupt(layer)
    X, Y, ids = U.dev_inputs(wl)
    layer.err.zero_()
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    return Yc, Y.cpu().numpy(), int(layer.err.item())


@pytest.mark.parametrize("kind", ["a_page_past_pool", "b_page_negative", "rank_above_64"])
@pytest.mark.parametrize("thresh", [None, 16])
def test_bad_page_skips_tokens_and_sets_bit(H, kind, thresh):
    """A page id outside the pool (or -1 inside the rank), or a rank above 64,
    written straight into the device tables: the kernels check every page before
    any load, leave that slot's rows at Y_base, set LORA_DEV_ERR_BAD_PAGE and
    give every other token the clean result bit for bit.  thresh = 16 puts the
    long runs on the tensor-core tiles."""
    if thresh is None:
        wl = W.random_small(seed=71, T=60, d_in=256, d_out=200, S=6, ranks=(16, 33, 64), p_none=0.0)
    else:
        wl = W.segments(72, [40, 200, 17, 130], 256, 200, S=6, ranks=(16, 33, 64))
    bad_slot = int(wl.ids[len(wl.ids) // 2])

    def corrupt(layer):
        if kind == "a_page_past_pool":
            layer.page_table[bad_slot, 0, 0] = H.lora_pool_num_pages(layer.pool_a) + 3
        elif kind == "b_page_negative":
            layer.page_table[bad_slot, 1, 0] = -1
        else:
            layer.ranks[bad_slot] = 65

    Yc, Yb, err = _corrupt_and_apply(H, wl, corrupt, thresh)
    assert err == H.DEV_ERR_BAD_PAGE
    rows = wl.ids == bad_slot
    assert rows.any() and (~rows).any()
    assert np.array_equal(Yb[rows], wl.Y_base[rows])
    assert np.array_equal(Yb[~rows], Yc[~rows])


def test_distinct_scales_reach_every_slot(H):
    """Every slot carries its own alpha / r, and the result of each slot's tokens
    follows that slot's scale: rescaling one slot's alpha changes only its rows,
    by exactly the expected factor within the tolerance."""
    import torch
    wl = W.random_small(seed=73, T=48, d_in=128, d_out=96, S=8, ranks=(4, 16, 33), p_none=0.0)
    sc = wl.scales_f32()
    used = np.unique(wl.ids)
    assert len(np.unique(sc[used])) >= 3           # the generator gives slots different scales
    Y1, err, layer = _run_apply(H, wl)
    assert err == 0
    ref, _ = U.oracle_full(wl)
    U.assert_parity(Y1, ref, wl.Y_base)
    k = int(used[0])
    layer.scales[k] = float(sc[k]) * 3.0
    X, Y, ids = U.dev_inputs(wl)
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    Y2 = Y.cpu().numpy()
    rows = wl.ids == k
    assert np.array_equal(Y2[~rows], Y1[~rows])
    d1 = Y1[rows].astype(np.float64) - wl.Y_base[rows]
    d2 = Y2[rows].astype(np.float64) - wl.Y_base[rows]
    assert np.abs(d2 - 3.0 * d1).max() <= 1e-4 * np.abs(d1).max() + 1e-6


_PLANNED_CASES = {
    "decode_q_proj_7b": lambda: W.by_name("decode_q_proj_7b"),
    "mixed_mlp_up": lambda: W.by_name("mixed_mlp_up"),
    "tiny": lambda: W.by_name("tiny"),
    # long runs: the tile launches, whose per-tile quarter counters must be back
    # at 0 for the next layer over the same plan
    "segments": lambda: W.segments(8, [300, 7, 129, 40, 256], 512, 1024, S=6),
}


@pytest.mark.parametrize("name", sorted(_PLANNED_CASES))
@pytest.mark.parametrize("path", ["cluster", "split"])
def test_planned_layers_after_one_plan_bit_exact(H, name, path):
    """One plan, then several layers on the same stream: every layer after the
    first starts while the previous one drains and reads the plan (and, on the
    cluster path, the adapter pages) before its grid-dependency wait.  Each layer
    must equal the one-call lora_apply on its own inputs, bit for bit, and the
    oracle."""
    import torch
    old = H.lora_get_option(H.OPT_GATHER_PATH)
    H.lora_set_option(H.OPT_GATHER_PATH, H.GATHER_CLUSTER if path == "cluster" else H.GATHER_SPLIT)
    try:
        wl = _PLANNED_CASES[name]()
        layers = [U.make_layer(wl) for _ in range(3)]
        X, _, ids = U.dev_inputs(wl)
        Ys = [U.dev_inputs(wl)[1] for _ in layers]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            layers[0].plan(ids, stream=stream)
            for lay, Y in zip(layers, Ys):
                lay.apply_planned(X, Y, stream=stream, ws=layers[0].ws)
        torch.cuda.synchronize()
        ref_one, _, _ = _run_apply(H, wl)
        oracle, _ = U.oracle_full(wl)
        for lay, Y in zip(layers, Ys):
            assert int(lay.err.item()) == 0
            y = Y.cpu().numpy()
            assert np.array_equal(y, ref_one)
            U.assert_parity(y, oracle, wl.Y_base,
                            delta_rel=U.DELTA_REL_TENSOR if name == "segments" else U.DELTA_REL_GATHER)
    finally:
        H.lora_set_option(H.OPT_GATHER_PATH, old)
