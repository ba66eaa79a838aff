"""lora_apply_noalloc: the fused call for callers that cannot allocate device memory.

Some users of the library cannot hand it a workspace: a plug-in running inside
a host framework that owns all device memory through its own pool, or a
serving loop that must not call cudaMalloc/cudaFree because those calls can
synchronise the device.  lora_apply_noalloc keeps the plan in a fixed scratch
array inside the library instead.  These tests check, through the C ABI, that
it gives the same Y as lora_apply bit for bit (the two run the same kernels on
the same plan) and matches the fp64 oracle, on calls in a row with different
batches (so stale scratch contents from an earlier call would show), that the
tensor-core launch really runs for a batch with long runs, that the largest
batch it admits (LORA_NOALLOC_MAX_TOKENS tokens, LORA_MAX_SLOTS slots) fits its
scratch, and that larger sizes are refused before any work is queued.

This file is collected last so that a run stopping at the first failure has
run every other test before it.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from tests import _util as U


def _defaults(H):
    H.lora_set_option(H.OPT_LONG_SEGMENT, 128)
    H.lora_set_option(H.OPT_DECODE_JOB_TOKENS, H.MAX_JOB_TOKENS)


def _compare_with_apply(H, wl, launches=None, delta_rel=U.DELTA_REL_GATHER):
    import torch
    layer = U.make_layer(wl)
    X, Y_ref, ids = U.dev_inputs(wl)
    Y_new = Y_ref.clone()
    err_new = torch.zeros(1, dtype=torch.int32, device="cuda")
    layer.err.zero_()
    layer.apply(X, Y_ref, ids)                                   # existing entry point
    H.lora_apply_noalloc(X, Y_new, wl.T, wl.d_in, wl.d_out, ids, wl.S, layer.ranks, layer.scales,
                         layer.page_table, layer.pool_a, layer.pool_b, err_new)
    n_launch = H.lora_last_launch_count()
    torch.cuda.synchronize()
    a = Y_ref.cpu().numpy()
    b = Y_new.cpu().numpy()
    assert int(err_new.item()) == int(layer.err.item()) == 0
    assert np.array_equal(a, b)                                  # same kernels, same plan
    assert not np.array_equal(b, wl.Y_base)                      # the call did change Y
    ref, rerr = U.oracle_full(wl)
    assert rerr == 0
    U.assert_parity(b, ref, wl.Y_base, delta_rel=delta_rel)
    if launches is not None:
        assert n_launch == launches
    return n_launch


@pytest.mark.gpu
def test_noalloc_matches_lora_apply_on_calls_in_a_row():
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    _defaults(H)
    # first call: a decode batch (plan + gather kernel)
    _compare_with_apply(H, W.decode_q_proj_7b(), launches=2)
    # second call: a different batch with long contiguous segments (plan +
    # gather + tensor-core tiles)
    _compare_with_apply(H, W.segments(8, [300, 7, 129, 40], 512, 1024, S=6), launches=3,
                        delta_rel=U.DELTA_REL_TENSOR)
    # third call: back to a small decode batch over the now-larger stale scratch
    _compare_with_apply(H, W.random_small(seed=81, T=33, d_in=264, d_out=136, S=9), launches=2)


@pytest.mark.gpu
def test_noalloc_largest_admitted_batch():
    """T = LORA_NOALLOC_MAX_TOKENS tokens over LORA_MAX_SLOTS slots: the plan of the
    largest call the entry point admits fits its fixed scratch."""
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    _defaults(H)
    wl = W.random_small(seed=82, T=H.NOALLOC_MAX_TOKENS, d_in=64, d_out=72, S=H.MAX_SLOTS,
                        ranks=(1, 4, 16, 64), p_none=0.05)
    _compare_with_apply(H, wl)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    """Validation happens on the host before any CUDA call, so this runs without a GPU."""
    import heterogeneous_adapter_batching_b200 as H
    from heterogeneous_adapter_batching_b200 import build
    build.build()
    lib = H.load_library()
    fake = ctypes.c_void_p(0x7F0000000000)
    pool = ctypes.c_void_p()
    assert lib.lora_pool_create(fake, 16 * 64 * 2 * 4, 64, 16, ctypes.byref(pool)) == 0
    try:
        rc = lib.lora_apply_noalloc(fake, fake, H.NOALLOC_MAX_TOKENS + 1, 64, 64, fake, 4, fake, fake, fake,
                                    pool, pool, None, None)
        assert rc == -8
        rc = lib.lora_apply_noalloc(fake, fake, 16, 64, 64, fake, H.MAX_SLOTS + 1, fake, fake, fake,
                                    pool, pool, None, None)
        assert rc == -1
    finally:
        lib.lora_pool_destroy(pool)
