"""CPU-only checks of the C-ABI library: it loads, exports every declared
symbol, and its host-side logic (validation, pool free list, options,
workspace sizing) behaves as include/lora.h states.  No compute call is made."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora.h")


@pytest.fixture(scope="module")
def lib():
    from heterogeneous_adapter_batching_b200 import build
    build.build()
    import heterogeneous_adapter_batching_b200 as H
    return H.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    import heterogeneous_adapter_batching_b200 as H
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(H.EXPORTS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", H.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (lora_\w+)", out))
    assert set(names) <= exported


def test_missing_library_fails_loudly(tmp_path):
    from heterogeneous_adapter_batching_b200 import _binding
    saved = _binding._lib
    _binding._lib = None
    try:
        with pytest.raises(OSError):
            _binding.load_library(str(tmp_path / "nope.so"))
    finally:
        _binding._lib = saved


FAKE_DEV = 0x7F0000000000   # aligned address; the pool never dereferences it on the host


def _pool(lib, nbytes, width, rows=16, addr=FAKE_DEV):
    out = ctypes.c_void_p()
    rc = lib.lora_pool_create(ctypes.c_void_p(addr), nbytes, width, rows, ctypes.byref(out))
    return rc, out


def test_pool_create_validation(lib):
    rc, p = _pool(lib, 16 * 64 * 2 * 10 + 5, 64)
    assert rc == 0
    assert lib.lora_pool_num_pages(p) == 10 and lib.lora_pool_free_pages(p) == 10
    assert lib.lora_pool_destroy(p) == 0
    assert _pool(lib, 1 << 20, 60)[0] == -1         # width not a multiple of 8
    assert _pool(lib, 1 << 20, 64, rows=8)[0] == -1  # page rows must be 16
    assert _pool(lib, 1 << 20, 64, addr=FAKE_DEV + 16)[0] == -1  # misaligned
    assert _pool(lib, 100, 64)[0] == -1             # less than one page
    assert lib.lora_pool_free_pages(None) == -1 and lib.lora_pool_num_pages(None) == -1


def test_load_and_apply_validation_before_any_cuda_call(lib):
    rc, pa = _pool(lib, 16 * 64 * 2 * 8, 64)
    rc2, pb = _pool(lib, 16 * 32 * 2 * 8, 32, addr=FAKE_DEV + (1 << 20))
    assert rc == rc2 == 0
    fake = ctypes.c_void_p(FAKE_DEV + (2 << 20))
    s = None
    # rank outside [1, 64]
    assert lib.lora_pool_load(pa, pb, 0, 4, 0, 1.0, fake, fake, None, fake, fake, fake, s) == -2
    assert lib.lora_pool_load(pa, pb, 0, 4, 65, 1.0, fake, fake, None, fake, fake, fake, s) == -2
    # slot outside [0, S)
    assert lib.lora_pool_load(pa, pb, 4, 4, 8, 1.0, fake, fake, None, fake, fake, fake, s) == -5
    assert lib.lora_pool_load(pa, pb, -1, 4, 8, 1.0, fake, fake, None, fake, fake, fake, s) == -5
    # NULL pointers
    assert lib.lora_pool_load(pa, pb, 0, 4, 8, 1.0, None, fake, None, fake, fake, fake, s) == -1
    # evicting a slot that holds nothing
    assert lib.lora_pool_evict(pa, pb, 0, 4, fake, fake, fake, s) == -5
    ws_n = lib.lora_workspace_size(8, 4)
    ws = ctypes.c_void_p(FAKE_DEV + (4 << 20))
    # widths must match the pools
    assert lib.lora_apply(fake, fake, 8, 64, 64, fake, 4, fake, fake, fake, pa, pb, ws, ws_n, None, s) == -3
    assert lib.lora_apply(fake, fake, 8, 32, 32, fake, 4, fake, fake, fake, pa, pb, ws, ws_n, None, s) == -3
    # workspace too small / missing
    assert lib.lora_apply(fake, fake, 8, 64, 32, fake, 4, fake, fake, fake, pa, pb, ws, ws_n - 1, None, s) == -7
    assert lib.lora_apply(fake, fake, 8, 64, 32, fake, 4, fake, fake, fake, pa, pb, None, ws_n, None, s) == -7
    # bad sizes
    assert lib.lora_apply(fake, fake, -1, 64, 32, fake, 4, fake, fake, fake, pa, pb, ws, ws_n, None, s) == -1
    assert lib.lora_apply(fake, fake, 8, 64, 32, fake, 0, fake, fake, fake, pa, pb, ws, ws_n, None, s) == -1
    assert lib.lora_apply(fake, fake, 8, 64, 32, fake, 4097, fake, fake, fake, pa, pb, ws, ws_n, None, s) == -1
    # an empty batch is a no-op that launches nothing
    assert lib.lora_apply(fake, fake, 0, 64, 32, fake, 4, fake, fake, fake, pa, pb, ws,
                          lib.lora_workspace_size(0, 4), None, s) == 0
    # lora_apply_multi: projection count, per-projection widths and workspace
    from heterogeneous_adapter_batching_b200._binding import LoraProjection
    good = LoraProjection(FAKE_DEV + (2 << 20), 32, FAKE_DEV + (2 << 20), FAKE_DEV + (2 << 20),
                          FAKE_DEV + (2 << 20), pa.value, pb.value)
    wrong = LoraProjection(FAKE_DEV + (2 << 20), 64, FAKE_DEV + (2 << 20), FAKE_DEV + (2 << 20),
                           FAKE_DEV + (2 << 20), pa.value, pb.value)
    arr = (LoraProjection * 9)(*([good] * 9))
    assert lib.lora_apply_multi(fake, 8, 64, fake, 4, arr, 0, ws, ws_n, None, s) == -1
    assert lib.lora_apply_multi(fake, 8, 64, fake, 4, arr, 9, ws, ws_n, None, s) == -1
    assert lib.lora_apply_multi(fake, 8, 64, fake, 4, None, 1, ws, ws_n, None, s) == -1
    assert lib.lora_apply_multi(fake, 8, 64, fake, 4, arr, 2, ws, ws_n - 1, None, s) == -7
    two = (LoraProjection * 2)(good, wrong)
    assert lib.lora_apply_multi(fake, 8, 64, fake, 4, two, 2, ws, ws_n, None, s) == -3
    assert lib.lora_apply_multi(fake, 8, 32, fake, 4, arr, 1, ws, ws_n, None, s) == -3
    assert lib.lora_apply_multi(fake, 0, 64, fake, 4, arr, 8, ws, lib.lora_workspace_size(0, 4), None, s) == 0
    assert lib.lora_last_launch_count() == 0
    assert lib.lora_shrink(fake, 8, 32, fake, 4, fake, fake, pa, fake, ws, ws_n, None, s) == -3
    assert lib.lora_expand_add(fake, fake, 8, 64, fake, 4, fake, fake, fake, pb, ws, ws_n, None, s) == -3
    # the strided expand: the pool's width must be d_out, the row stride >= d_out and a multiple of 4
    assert lib.lora_expand_add_strided(fake, fake, 64, 8, 64, fake, 4, fake, fake, fake, pb, ws, ws_n, None, s) == -3
    assert lib.lora_expand_add_strided(fake, fake, 30, 8, 32, fake, 4, fake, fake, fake, pb, ws, ws_n, None, s) == -1
    assert lib.lora_expand_add_strided(fake, fake, 34, 8, 32, fake, 4, fake, fake, fake, pb, ws, ws_n, None, s) == -1
    assert lib.lora_last_launch_count() == 0
    lib.lora_pool_destroy(pa)
    lib.lora_pool_destroy(pb)


def test_workspace_size(lib):
    prev = 0
    for T in (0, 1, 7, 64, 1000, 17000):
        n = lib.lora_workspace_size(T, 32)
        assert n % 256 == 0 and n >= prev
        assert n >= 4 * T + 16 * 2 * T
        prev = n
    assert lib.lora_workspace_size(-1, 4) == 0 and lib.lora_workspace_size(4, 0) == 0


def test_options(lib):
    old1, old2 = lib.lora_get_option(1), lib.lora_get_option(2)
    try:
        assert lib.lora_set_option(1, 0) == 0 and lib.lora_get_option(1) == 0
        assert lib.lora_set_option(1, -1) == -1
        assert lib.lora_set_option(2, 17) == -1 and lib.lora_set_option(2, 0) == -1
        assert lib.lora_set_option(2, 16) == 0 and lib.lora_get_option(2) == 16
        assert lib.lora_set_option(2, 3) == 0 and lib.lora_get_option(2) == 3
        assert lib.lora_set_option(99, 1) == -1 and lib.lora_get_option(99) == -1
    finally:
        lib.lora_set_option(1, old1)
        lib.lora_set_option(2, old2)
