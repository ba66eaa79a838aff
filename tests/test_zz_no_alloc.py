"""lora_apply_noalloc: the fused call for callers that cannot allocate device memory.

Some users of the library cannot hand it a workspace: a plug-in running inside
a host framework that owns all device memory through its own pool, or a
serving loop that must not call cudaMalloc/cudaFree because those calls can
synchronise the device.  lora_apply_noalloc keeps the plan in a fixed scratch
array inside the library instead.  These tests check, through the C ABI, that
it gives the same Y as lora_apply on two calls in a row (the second one on a
different batch, so stale scratch contents from the first would show), and
that sizes beyond its fixed scratch are refused before any work is queued.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from tests import _util as U


def _compare_with_apply(H, wl):
    import torch
    layer = U.make_layer(wl)
    X, Y_ref, ids = U.dev_inputs(wl)
    Y_new = Y_ref.clone()
    err_new = torch.zeros(1, dtype=torch.int32, device="cuda")
    layer.err.zero_()
    layer.apply(X, Y_ref, ids)                                   # existing entry point
    H.lora_apply_noalloc(X, Y_new, wl.T, wl.d_in, wl.d_out, ids, wl.S, layer.ranks, layer.scales,
                         layer.page_table, layer.pool_a, layer.pool_b, err_new)
    torch.cuda.synchronize()
    a = Y_ref.cpu().numpy().astype(np.float64)
    b = Y_new.cpu().numpy().astype(np.float64)
    assert int(err_new.item()) == int(layer.err.item()) == 0
    assert (np.abs(b - a) <= U.ATOL + U.RTOL * np.abs(a)).all()
    assert not np.array_equal(a, wl.Y_base)                      # the call did change Y


@pytest.mark.gpu
def test_noalloc_matches_lora_apply_on_two_calls():
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    # first call: a decode batch (gather kernels)
    _compare_with_apply(H, W.decode_q_proj_7b())
    # second call: a different batch with long contiguous segments (tensor-core tiles)
    _compare_with_apply(H, W.segments(8, [300, 7, 129, 40], 512, 1024, S=6))


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
    finally:
        lib.lora_pool_destroy(pool)
