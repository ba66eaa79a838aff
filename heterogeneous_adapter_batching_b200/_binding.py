"""ctypes binding of liblora (include/lora.h): argument marshalling only.

Every function has the name of the C entry point it calls and takes torch
tensors (device memory) or plain Python numbers; it passes their pointers
and sizes through and raises LoraError on a negative return code.  There is
no fallback: if liblora.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblora.so")

LORA_OK = 0
ERR_NAMES = {
    -1: "LORA_ERR_INVALID_ARG", -2: "LORA_ERR_BAD_RANK", -3: "LORA_ERR_WIDTH_MISMATCH",
    -4: "LORA_ERR_POOL_OOM", -5: "LORA_ERR_BAD_SLOT", -6: "LORA_ERR_CUDA", -7: "LORA_ERR_WORKSPACE",
    -8: "LORA_ERR_TOO_LARGE", -9: "LORA_ERR_ALL_PINNED",
}
DEV_ERR_BAD_ID = 1
DEV_ERR_EMPTY_SLOT = 2
DEV_ERR_TIMEOUT = 4
DEV_ERR_BAD_PAGE = 8
PAGE_ROWS = 16
MAX_RANK = 64
MAX_PAGES_PER_MATRIX = 4
MAX_SLOTS = 4096
OPT_LONG_SEGMENT = 1
OPT_DECODE_JOB_TOKENS = 2
OPT_GATHER_PATH = 3
GATHER_AUTO, GATHER_CLUSTER, GATHER_SPLIT = 0, 1, 2
OPT_PLAN_KERNEL = 4
PLAN_AUTO, PLAN_GENERAL = 0, 1
NOALLOC_MAX_TOKENS = 32768
NOALLOC_SCRATCH_BYTES = 2162688
MAX_JOB_TOKENS = 16
MAX_PROJECTIONS = 8

EXPORTS = [
    "lora_pool_create", "lora_pool_destroy", "lora_pool_free_pages", "lora_pool_num_pages",
    "lora_pool_alloc_pages", "lora_pool_free_page_list", "lora_pool_usage",
    "lora_pool_load", "lora_pool_evict", "lora_pool_read_row", "lora_workspace_size",
    "lora_plan", "lora_shrink", "lora_expand_add", "lora_expand_add_strided", "lora_apply", "lora_apply_planned", "lora_apply_noalloc",
    "lora_apply_multi", "lora_apply_multi_planned",
    "lora_slot_cache_create", "lora_slot_cache_destroy", "lora_slot_cache_acquire", "lora_slot_cache_unpin",
    "lora_slot_cache_invalidate", "lora_slot_cache_lookup", "lora_slot_cache_stats",
    "lora_set_option", "lora_get_option", "lora_last_cuda_error", "lora_last_launch_count",
]


class LoraProjection(ctypes.Structure):
    """lora_projection_t: one projection of lora_apply_multi."""
    _fields_ = [("Y", ctypes.c_void_p), ("d_out", ctypes.c_int), ("ranks", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("page_table", ctypes.c_void_p), ("pa", ctypes.c_void_p),
                ("pb", ctypes.c_void_p)]


class LoraError(RuntimeError):
    def __init__(self, name: str, rc: int, detail: str = ""):
        self.rc = rc
        super().__init__(f"{name} failed: {ERR_NAMES.get(rc, rc)}{(' (' + detail + ')') if detail else ''}")


_lib = None
V = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
Z = ctypes.c_size_t


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblora.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"liblora.so not found at {path}; run heterogeneous_adapter_batching_b200.build.build()")
    lib = ctypes.CDLL(path)
    sig = {
        "lora_pool_create": (I, [V, Z, I, I, ctypes.POINTER(V)]),
        "lora_pool_destroy": (I, [V]),
        "lora_pool_free_pages": (I, [V]),
        "lora_pool_num_pages": (I, [V]),
        "lora_pool_alloc_pages": (I, [V, I, V]),
        "lora_pool_free_page_list": (I, [V, V, I]),
        "lora_pool_usage": (I, [V, ctypes.POINTER(I), ctypes.POINTER(I)]),
        "lora_pool_load": (I, [V, V, I, I, I, F, V, V, V, V, V, V, V]),
        "lora_pool_evict": (I, [V, V, I, I, V, V, V, V]),
        "lora_pool_read_row": (I, [V, V, I, I, I, I, V, V]),
        "lora_workspace_size": (Z, [I, I]),
        "lora_plan": (I, [V, I, V, I, V, V, V, Z, V, V]),
        "lora_shrink": (I, [V, I, I, V, I, V, V, V, V, V, Z, V, V]),
        "lora_expand_add": (I, [V, V, I, I, V, I, V, V, V, V, V, Z, V, V]),
        "lora_expand_add_strided": (I, [V, V, I, I, I, V, I, V, V, V, V, V, Z, V, V]),
        "lora_apply": (I, [V, V, I, I, I, V, I, V, V, V, V, V, V, Z, V, V]),
        "lora_apply_planned": (I, [V, V, I, I, I, I, V, V, V, V, V, V, Z, V, V]),
        "lora_apply_noalloc": (I, [V, V, I, I, I, V, I, V, V, V, V, V, V, V]),
        "lora_apply_multi": (I, [V, I, I, V, I, ctypes.POINTER(LoraProjection), I, V, Z, V, V]),
        "lora_apply_multi_planned": (I, [V, I, I, I, ctypes.POINTER(LoraProjection), I, V, Z, V, V]),
        "lora_slot_cache_create": (I, [I, ctypes.POINTER(V)]),
        "lora_slot_cache_destroy": (I, [V]),
        "lora_slot_cache_acquire": (I, [V, ctypes.c_int64, I, ctypes.POINTER(I), ctypes.POINTER(I),
                                        ctypes.POINTER(ctypes.c_int64)]),
        "lora_slot_cache_unpin": (I, [V, I]),
        "lora_slot_cache_invalidate": (I, [V, I]),
        "lora_slot_cache_lookup": (I, [V, ctypes.c_int64, ctypes.POINTER(I)]),
        "lora_slot_cache_stats": (I, [V, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                      ctypes.POINTER(ctypes.c_int64)]),
        "lora_set_option": (I, [I, I]),
        "lora_get_option": (I, [I]),
        "lora_last_cuda_error": (ctypes.c_char_p, []),
        "lora_last_launch_count": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(name: str, rc: int):
    if rc != LORA_OK:
        detail = lora_last_cuda_error() if rc == -6 else ""
        raise LoraError(name, rc, detail)
    return rc


class Pool:
    """Host handle of one page pool over a caller-owned device buffer."""

    def __init__(self, handle: int, buf: torch.Tensor, width: int):
        self.handle = handle
        self.buf = buf          # keeps the device memory alive
        self.width = width

    def __del__(self):
        try:
            if self.handle and _lib is not None:
                _lib.lora_pool_destroy(ctypes.c_void_p(self.handle))
                self.handle = 0
        except Exception:
            pass

    @property
    def _h(self):
        return ctypes.c_void_p(self.handle)


def lora_pool_create(dev_buf: torch.Tensor, width: int, page_rows: int = PAGE_ROWS) -> Pool:
    lib = load_library()
    out = ctypes.c_void_p()
    nbytes = dev_buf.numel() * dev_buf.element_size()
    _check("lora_pool_create", lib.lora_pool_create(_p(dev_buf), nbytes, width, page_rows, ctypes.byref(out)))
    return Pool(out.value, dev_buf, width)


def lora_pool_destroy(pool: Pool) -> None:
    if pool.handle:
        load_library().lora_pool_destroy(pool._h)
        pool.handle = 0


def lora_pool_free_pages(pool: Pool) -> int:
    return load_library().lora_pool_free_pages(pool._h)


def lora_pool_num_pages(pool: Pool) -> int:
    return load_library().lora_pool_num_pages(pool._h)


def lora_pool_alloc_pages(pool: Pool, n: int) -> torch.Tensor:
    """n free pages of the pool for another tenant (KV blocks); host int32 ids."""
    ids = torch.empty(max(n, 0), dtype=torch.int32)
    _check("lora_pool_alloc_pages", load_library().lora_pool_alloc_pages(pool._h, n, _p(ids) if n > 0 else None))
    return ids


def lora_pool_free_page_list(pool: Pool, ids: torch.Tensor) -> None:
    ids = ids.to(torch.int32).contiguous()
    assert ids.device.type == "cpu"
    _check("lora_pool_free_page_list", load_library().lora_pool_free_page_list(
        pool._h, _p(ids) if ids.numel() else None, ids.numel()))


def lora_pool_usage(pool: Pool):
    """(pages held by adapters, pages held through lora_pool_alloc_pages)."""
    a, o = ctypes.c_int(), ctypes.c_int()
    _check("lora_pool_usage", load_library().lora_pool_usage(pool._h, ctypes.byref(a), ctypes.byref(o)))
    return a.value, o.value


def lora_pool_load(pa: Pool, pb: Pool, slot: int, num_slots: int, rank: int, alpha: float,
                   a_t: torch.Tensor, b: torch.Tensor, page_ids: Optional[torch.Tensor],
                   page_table: torch.Tensor, scales: torch.Tensor, ranks: torch.Tensor, stream=None) -> None:
    """a_t: [rank, d_in] bf16 (host or device), b: [rank, d_out] bf16; page_ids: host int32 [2, 4] or None."""
    if page_ids is not None:
        assert page_ids.device.type == "cpu" and page_ids.dtype == torch.int32 and page_ids.is_contiguous()
    _check("lora_pool_load", load_library().lora_pool_load(
        pa._h, pb._h, slot, num_slots, rank, alpha, _p(a_t), _p(b), _p(page_ids),
        _p(page_table), _p(scales), _p(ranks), _s(stream)))


def lora_pool_evict(pa: Pool, pb: Pool, slot: int, num_slots: int, page_table: torch.Tensor,
                    scales: torch.Tensor, ranks: torch.Tensor, stream=None) -> None:
    _check("lora_pool_evict", load_library().lora_pool_evict(
        pa._h, pb._h, slot, num_slots, _p(page_table), _p(scales), _p(ranks), _s(stream)))


def lora_pool_read_row(pool: Pool, page_table: torch.Tensor, num_slots: int, slot: int, m: int, k: int,
                       out: torch.Tensor, stream=None) -> None:
    _check("lora_pool_read_row", load_library().lora_pool_read_row(
        pool._h, _p(page_table), num_slots, slot, m, k, _p(out), _s(stream)))


def lora_workspace_size(T: int, num_slots: int) -> int:
    return int(load_library().lora_workspace_size(T, num_slots))


def lora_plan(ids, T, ranks, num_slots, perm_out, seg_start_out, ws, err=None, stream=None) -> None:
    _check("lora_plan", load_library().lora_plan(
        _p(ids), T, _p(ranks), num_slots, _p(perm_out), _p(seg_start_out), _p(ws),
        ws.numel() * ws.element_size(), _p(err), _s(stream)))


def lora_shrink(X, T, d_in, ids, num_slots, ranks, page_table, pa: Pool, V, ws, err=None, stream=None) -> None:
    _check("lora_shrink", load_library().lora_shrink(
        _p(X), T, d_in, _p(ids), num_slots, _p(ranks), _p(page_table), pa._h, _p(V), _p(ws),
        ws.numel() * ws.element_size(), _p(err), _s(stream)))


def lora_expand_add(V, Y, T, d_out, ids, num_slots, ranks, scales, page_table, pb: Pool, ws, err=None,
                    stream=None) -> None:
    _check("lora_expand_add", load_library().lora_expand_add(
        _p(V), _p(Y), T, d_out, _p(ids), num_slots, _p(ranks), _p(scales), _p(page_table), pb._h, _p(ws),
        ws.numel() * ws.element_size(), _p(err), _s(stream)))


def lora_expand_add_strided(V, Y, ldy, T, d_out, ids, num_slots, ranks, scales, page_table, pb: Pool, ws, err=None,
                            stream=None) -> None:
    """Y: a [T, d_out] column block of a wider fp32 tensor whose rows are ldy apart."""
    _check("lora_expand_add_strided", load_library().lora_expand_add_strided(
        _p(V), _p(Y), ldy, T, d_out, _p(ids), num_slots, _p(ranks), _p(scales), _p(page_table), pb._h, _p(ws),
        ws.numel() * ws.element_size(), _p(err), _s(stream)))


def lora_apply(X, Y, T, d_in, d_out, ids, num_slots, ranks, scales, page_table, pa: Pool, pb: Pool, ws,
               err=None, stream=None) -> None:
    _check("lora_apply", load_library().lora_apply(
        _p(X), _p(Y), T, d_in, d_out, _p(ids), num_slots, _p(ranks), _p(scales), _p(page_table),
        pa._h, pb._h, _p(ws), ws.numel() * ws.element_size(), _p(err), _s(stream)))


def lora_apply_planned(X, Y, T, d_in, d_out, num_slots, ranks, scales, page_table, pa: Pool, pb: Pool, ws,
                       err=None, stream=None) -> None:
    _check("lora_apply_planned", load_library().lora_apply_planned(
        _p(X), _p(Y), T, d_in, d_out, num_slots, _p(ranks), _p(scales), _p(page_table),
        pa._h, pb._h, _p(ws), ws.numel() * ws.element_size(), _p(err), _s(stream)))


def lora_apply_noalloc(X, Y, T, d_in, d_out, ids, num_slots, ranks, scales, page_table, pa: Pool, pb: Pool,
                       err=None, stream=None) -> None:
    """lora_apply without a workspace: the plan lives in the library's fixed device
    scratch, for callers that cannot allocate device memory (see include/lora.h)."""
    _check("lora_apply_noalloc", load_library().lora_apply_noalloc(
        _p(X), _p(Y), T, d_in, d_out, _p(ids), num_slots, _p(ranks), _p(scales), _p(page_table),
        pa._h, pb._h, _p(err), _s(stream)))


def _proj_array(projs):
    arr = (LoraProjection * len(projs))()
    for i, (Y, d_out, ranks, scales, page_table, pa, pb) in enumerate(projs):
        arr[i] = LoraProjection(Y.data_ptr(), d_out, ranks.data_ptr(), scales.data_ptr(), page_table.data_ptr(),
                                pa.handle, pb.handle)
    return arr


def lora_apply_multi(X, T, d_in, ids, num_slots, projs, ws, err=None, stream=None) -> None:
    """projs: sequence of (Y, d_out, ranks, scales, page_table, pa: Pool, pb: Pool)."""
    _check("lora_apply_multi", load_library().lora_apply_multi(
        _p(X), T, d_in, _p(ids), num_slots, _proj_array(projs), len(projs), _p(ws), ws.numel() * ws.element_size(),
        _p(err), _s(stream)))


def lora_apply_multi_planned(X, T, d_in, num_slots, projs, ws, err=None, stream=None) -> None:
    _check("lora_apply_multi_planned", load_library().lora_apply_multi_planned(
        _p(X), T, d_in, num_slots, _proj_array(projs), len(projs), _p(ws), ws.numel() * ws.element_size(),
        _p(err), _s(stream)))


class SlotCache:
    """lora_slot_cache_t: which adapter key lives in which slot (exact LRU over
    the slots no running batch pins).  Host bookkeeping only."""

    def __init__(self, num_slots: int):
        h = ctypes.c_void_p()
        _check("lora_slot_cache_create", load_library().lora_slot_cache_create(num_slots, ctypes.byref(h)))
        self.handle = h.value
        self.num_slots = num_slots
        self._slot, self._hit, self._ev = ctypes.c_int(), ctypes.c_int(), ctypes.c_int64()

    def __del__(self):
        try:
            if self.handle and _lib is not None:
                _lib.lora_slot_cache_destroy(ctypes.c_void_p(self.handle))
                self.handle = 0
        except Exception:
            pass

    def acquire(self, key: int, pin: bool = False):
        """-> (slot, hit, evicted_key or -1)."""
        _check("lora_slot_cache_acquire", _lib.lora_slot_cache_acquire(
            ctypes.c_void_p(self.handle), key, 1 if pin else 0, ctypes.byref(self._slot), ctypes.byref(self._hit),
            ctypes.byref(self._ev)))
        return self._slot.value, bool(self._hit.value), self._ev.value

    def unpin(self, slot: int) -> None:
        _check("lora_slot_cache_unpin", _lib.lora_slot_cache_unpin(ctypes.c_void_p(self.handle), slot))

    def invalidate(self, slot: int) -> None:
        _check("lora_slot_cache_invalidate", _lib.lora_slot_cache_invalidate(ctypes.c_void_p(self.handle), slot))

    def lookup(self, key: int) -> int:
        _check("lora_slot_cache_lookup", _lib.lora_slot_cache_lookup(ctypes.c_void_p(self.handle), key,
                                                                     ctypes.byref(self._slot)))
        return self._slot.value

    def stats(self):
        h, m, e = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check("lora_slot_cache_stats", _lib.lora_slot_cache_stats(ctypes.c_void_p(self.handle), ctypes.byref(h),
                                                                   ctypes.byref(m), ctypes.byref(e)))
        return h.value, m.value, e.value


def lora_set_option(key: int, value: int) -> None:
    _check("lora_set_option", load_library().lora_set_option(key, value))


def lora_get_option(key: int) -> int:
    return int(load_library().lora_get_option(key))


def lora_last_cuda_error() -> str:
    return load_library().lora_last_cuda_error().decode()


def lora_last_launch_count() -> int:
    return int(load_library().lora_last_launch_count())
