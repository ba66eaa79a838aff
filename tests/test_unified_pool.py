"""Unified paging on the host: one free list of fixed-size pages serves adapter
weights and another tenant of the same memory (KV-cache blocks).

Page "Multi-LoRA Serving in Production", section "Unified Paging
Architecture": KV cache and adapter weights are pages of one pool, so memory
moves between them without external fragmentation.  The allocator needs no
GPU: the pool wraps a device address that is never dereferenced here.
"""
import ctypes

import numpy as np
import pytest

FAKE_DEV = 0x7F0000000000


@pytest.fixture(scope="module")
def lib():
    import heterogeneous_adapter_batching_b200 as H
    from heterogeneous_adapter_batching_b200 import build
    build.build()
    return H.load_library()


def _pool(lib, pages, width=64):
    h = ctypes.c_void_p()
    assert lib.lora_pool_create(ctypes.c_void_p(FAKE_DEV), pages * 16 * width * 2, width, 16, ctypes.byref(h)) == 0
    return h


def _alloc(lib, pool, n):
    ids = (ctypes.c_int32 * max(n, 1))()
    rc = lib.lora_pool_alloc_pages(pool, n, ids)
    return rc, list(ids)[:n]


def _free(lib, pool, ids):
    arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
    return lib.lora_pool_free_page_list(pool, arr, len(ids))


def _usage(lib, pool):
    a, o = ctypes.c_int(), ctypes.c_int()
    assert lib.lora_pool_usage(pool, ctypes.byref(a), ctypes.byref(o)) == 0
    return a.value, o.value


def test_alloc_free_accounting(lib):
    pool = _pool(lib, 64)
    try:
        rc, ids = _alloc(lib, pool, 10)
        assert rc == 0 and len(set(ids)) == 10 and all(0 <= i < 64 for i in ids)
        assert _usage(lib, pool) == (0, 10) and lib.lora_pool_free_pages(pool) == 54
        assert _free(lib, pool, ids[:5]) == 0
        assert _usage(lib, pool) == (0, 5) and lib.lora_pool_free_pages(pool) == 59
        assert _free(lib, pool, ids[:1]) == -5                      # already free
        assert _free(lib, pool, [ids[5], ids[5]]) == -5             # repeated: nothing returned
        assert _usage(lib, pool) == (0, 5)
        assert _free(lib, pool, [64]) == -5 and _free(lib, pool, [-1]) == -5
        rc, more = _alloc(lib, pool, 60)                            # 59 free
        assert rc == -4 and _usage(lib, pool) == (0, 5)             # nothing taken
        rc, more = _alloc(lib, pool, 59)
        assert rc == 0 and lib.lora_pool_free_pages(pool) == 0
        assert set(more).isdisjoint(ids[5:])
        assert _free(lib, pool, more + ids[5:]) == 0
        assert _usage(lib, pool) == (0, 0) and lib.lora_pool_free_pages(pool) == 64
        assert lib.lora_pool_alloc_pages(pool, -1, None) == -1
        assert lib.lora_pool_alloc_pages(pool, 0, None) == 0
    finally:
        lib.lora_pool_destroy(pool)


def test_random_interleaving_matches_a_model(lib):
    """Thousands of random takes and returns: never a page twice, counts always right."""
    rng = np.random.default_rng(5)
    N = 200
    pool = _pool(lib, N)
    held = []
    try:
        for _ in range(3000):
            if rng.random() < 0.55:
                n = int(rng.integers(0, 12))
                rc, ids = _alloc(lib, pool, n)
                if n <= N - len(held):
                    assert rc == 0 and not set(ids) & set(held)
                    held += ids
                else:
                    assert rc == -4
            elif held:
                k = int(rng.integers(1, min(len(held), 12) + 1))
                pick = [held[i] for i in rng.choice(len(held), size=k, replace=False)]
                assert _free(lib, pool, pick) == 0
                held = [h for h in held if h not in pick]
            assert _usage(lib, pool) == (0, len(held))
            assert lib.lora_pool_free_pages(pool) == N - len(held)
    finally:
        lib.lora_pool_destroy(pool)
