"""GPU parity of the tensor-core (tcgen05) path for long contiguous segments.

The long-segment threshold is lowered so that segments of every length take
the tile path, with ragged tails (tiles of fewer than 128 tokens), widths that
are not multiples of the 64-column blocks, ranks that are not multiples of the
16-row page, and a mix with short and non-contiguous segments (gather path).
Tolerance: |err| <= 2e-3 + 1e-2 |ref| per element, and the adapter delta within
2e-4 of its largest magnitude (v enters the second product as a bf16 high part and a
bf16 low part, about 16 significant bits).
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
    old = {k: H.lora_get_option(k) for k in (H.OPT_LONG_SEGMENT, H.OPT_DECODE_JOB_TOKENS)}
    yield
    for k, v in old.items():
        H.lora_set_option(k, v)


def _apply(wl, H=None):
    """Run lora_apply; when H is given also check the plan's job / tile counts."""
    import torch
    layer = U.make_layer(wl)
    X, Y, ids = U.dev_inputs(wl)
    layer.err.zero_()
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    if H is not None:
        lt = H.lora_get_option(H.OPT_LONG_SEGMENT)
        jmax = H.lora_get_option(H.OPT_DECODE_JOB_TOKENS)
        jt = U.plan_job_tokens(layer.ws)
        assert jt in U.job_size_candidates(jmax)
        n_valid, n_seg, n_jobs, n_tiles = U.plan_counts(layer.ws)
        assert (n_jobs, n_tiles) == U.expected_work(wl.ids, wl.ranks(), lt, jt)
    return Y.cpu().numpy(), int(layer.err.item())


@pytest.mark.parametrize("thresh", [1, 16, 100])
@pytest.mark.parametrize("seed,lens,d_in,d_out", [
    (1, [128], 64, 64),
    (2, [1, 2, 127, 128, 129, 300], 256, 256),
    (3, [17, 250, 5, 64, 400], 200, 328),
    (4, [513, 7, 1000], 1032, 520),
    (5, [90, 33, 256, 256, 12], 4096, 4096),
    (6, [5000], 256, 512),
    # many tiles per CTA (whole tiles finished from tensor memory) with empty
    # quarters of d_in: one K block (quarters 0-2 empty), three (quarter 0 empty)
    (7, [20000], 64, 128),
    (8, [20000], 192, 128),
])
def test_tile_path_segments(H, thresh, seed, lens, d_in, d_out):
    H.lora_set_option(H.OPT_LONG_SEGMENT, thresh)
    wl = W.segments(seed, lens, d_in, d_out, S=max(8, len(lens)), ranks=(1, 4, 8, 15, 16, 17, 33, 48, 64))
    Y, err = _apply(wl, H)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)


def test_tile_path_with_shared_slots_and_none(H):
    """Slots reused by several sequences (non-contiguous -> gather) next to long
    contiguous ones (tiles), plus id = -1 tokens that must stay bit-exact."""
    import torch
    H.lora_set_option(H.OPT_LONG_SEGMENT, 8)
    wl = W.segments(6, [40, 200, 3, 130, 60, 9, 300], 512, 768, S=5, reuse=True)
    ids = wl.ids.copy()
    ids[[0, 45, 250, 600]] = -1
    wl.ids[:] = ids
    Y, err = _apply(wl, H)
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)
    none = ids == -1
    assert np.array_equal(Y[none], wl.Y_base[none])


def test_tile_and_gather_paths_agree_with_oracle(H):
    wl = W.segments(7, [300, 200, 100], 1024, 1024, S=4)
    ref, _ = U.oracle_full(wl)
    H.lora_set_option(H.OPT_LONG_SEGMENT, 16)
    Yt, e1 = _apply(wl, H)
    H.lora_set_option(H.OPT_LONG_SEGMENT, 0)
    Yg, e2 = _apply(wl, H)
    assert e1 == e2 == 0
    U.assert_parity(Yt, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)
    U.assert_parity(Yg, ref, wl.Y_base)


def test_prefill_config_tile_path(H):
    """The prefill workload (16 sequences of 128-2048 tokens, 6 adapters) through the
    default threshold, i.e. on the tensor-core tiles."""
    wl = W.prefill()
    Y, err = _apply(wl, H)
    assert U.expected_work(wl.ids, wl.ranks(), H.lora_get_option(H.OPT_LONG_SEGMENT), 4)[1] >= 130  # tiles run
    ref, rerr = U.oracle_full(wl)
    assert err == rerr == 0
    U.assert_parity(Y, ref, wl.Y_base, delta_rel=U.DELTA_REL_TENSOR)
