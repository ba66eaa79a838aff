"""Device state of one adapted projection: two page pools, the slot tables and
the workspace, held in torch tensors (device memory only; every computation
goes through the C-ABI calls in _binding)."""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B


class AdapterLayer:
    """Pools, page table [S, 2, 4], ranks [S], scales [S], error word and workspace.

    pool_a holds A^T rows (width d_in), pool_b holds B rows (width d_out); when
    d_in == d_out and `shared_pool` is set, one pool serves both.
    """

    def __init__(self, d_in: int, d_out: int, num_slots: int, pages_a: int, pages_b: int,
                 max_tokens: int, device="cuda", shared_pool: bool = False):
        self.d_in, self.d_out, self.S = d_in, d_out, num_slots
        self.device = torch.device(device)
        rows_a = pages_a * B.PAGE_ROWS
        self.buf_a = torch.empty((rows_a, d_in), dtype=torch.bfloat16, device=self.device)
        self.pool_a = B.lora_pool_create(self.buf_a, d_in)
        if shared_pool and d_in == d_out:
            self.buf_b, self.pool_b = self.buf_a, self.pool_a
        else:
            rows_b = pages_b * B.PAGE_ROWS
            self.buf_b = torch.empty((rows_b, d_out), dtype=torch.bfloat16, device=self.device)
            self.pool_b = B.lora_pool_create(self.buf_b, d_out)
        self.page_table = torch.full((num_slots, 2, B.MAX_PAGES_PER_MATRIX), -1, dtype=torch.int32,
                                     device=self.device)
        self.ranks = torch.zeros(num_slots, dtype=torch.int32, device=self.device)
        self.scales = torch.zeros(num_slots, dtype=torch.float32, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.max_tokens = max_tokens
        nbytes = B.lora_workspace_size(max_tokens, num_slots)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)

    def load(self, slot: int, rank: int, alpha: float, a_t_bits: torch.Tensor, b_bits: torch.Tensor,
             page_ids: Optional[torch.Tensor] = None, stream=None) -> None:
        """a_t_bits [rank, d_in], b_bits [rank, d_out]: bf16 tensors (host or device)."""
        B.lora_pool_load(self.pool_a, self.pool_b, slot, self.S, rank, alpha, a_t_bits.contiguous(),
                         b_bits.contiguous(), page_ids, self.page_table, self.scales, self.ranks, stream)

    def evict(self, slot: int, stream=None) -> None:
        B.lora_pool_evict(self.pool_a, self.pool_b, slot, self.S, self.page_table, self.scales, self.ranks,
                          stream)

    # Unified paging (shared_pool): KV-cache blocks and adapter pages from one free list.
    def alloc_pages(self, n: int) -> torch.Tensor:
        """n pages of pool_a for another tenant (KV blocks: 16 vectors of d_in values
        each, rows [16 p, 16 p + 16) of buf_a); host int32 page ids."""
        return B.lora_pool_alloc_pages(self.pool_a, n)

    def free_pages(self, ids: torch.Tensor) -> None:
        B.lora_pool_free_page_list(self.pool_a, ids)

    def page_rows(self, page: int) -> torch.Tensor:
        """The 16 rows of page `page` of pool_a (a view of buf_a)."""
        return self.buf_a[page * B.PAGE_ROWS:(page + 1) * B.PAGE_ROWS]

    def apply(self, X: torch.Tensor, Y: torch.Tensor, ids: torch.Tensor, stream=None) -> None:
        T = X.shape[0]
        assert T <= self.max_tokens
        B.lora_apply(X, Y, T, self.d_in, self.d_out, ids, self.S, self.ranks, self.scales, self.page_table,
                     self.pool_a, self.pool_b, self.ws, self.err, stream)

    def apply_planned(self, X: torch.Tensor, Y: torch.Tensor, ws: Optional[torch.Tensor] = None,
                      stream=None) -> None:
        """Compute half only, with the plan already in `ws` (default: this layer's workspace)."""
        B.lora_apply_planned(X, Y, X.shape[0], self.d_in, self.d_out, self.S, self.ranks, self.scales,
                             self.page_table, self.pool_a, self.pool_b, self.ws if ws is None else ws,
                             self.err, stream)

    def shrink(self, X: torch.Tensor, ids: torch.Tensor, V: torch.Tensor, stream=None) -> None:
        B.lora_shrink(X, X.shape[0], self.d_in, ids, self.S, self.ranks, self.page_table, self.pool_a, V,
                      self.ws, self.err, stream)

    def expand_add(self, V: torch.Tensor, Y: torch.Tensor, ids: torch.Tensor, stream=None) -> None:
        B.lora_expand_add(V, Y, V.shape[0], self.d_out, ids, self.S, self.ranks, self.scales,
                          self.page_table, self.pool_b, self.ws, self.err, stream)

    def plan(self, ids: torch.Tensor, perm: Optional[torch.Tensor] = None, seg_start: Optional[torch.Tensor] = None,
             ws: Optional[torch.Tensor] = None, stream=None) -> None:
        B.lora_plan(ids, ids.shape[0], self.ranks, self.S, perm, seg_start, self.ws if ws is None else ws,
                    self.err, stream)


def apply_multi(layers, X: torch.Tensor, Ys, ids: Optional[torch.Tensor], ws: Optional[torch.Tensor] = None,
                err: Optional[torch.Tensor] = None, stream=None) -> None:
    """One lora_apply_multi call over several AdapterLayer objects that read the
    same X (same d_in and slot count): Ys[p] += branch of layers[p].  The plan
    follows layers[0]'s ranks; ws and err default to layers[0]'s.  With
    ids=None the plan already in ws is used (lora_apply_multi_planned)."""
    l0 = layers[0]
    projs = [(Y, l.d_out, l.ranks, l.scales, l.page_table, l.pool_a, l.pool_b) for l, Y in zip(layers, Ys)]
    ws = l0.ws if ws is None else ws
    err = l0.err if err is None else err
    if ids is None:
        B.lora_apply_multi_planned(X, X.shape[0], l0.d_in, l0.S, projs, ws, err, stream)
    else:
        B.lora_apply_multi(X, X.shape[0], l0.d_in, ids, l0.S, projs, ws, err, stream)



class AdapterCache:
    """A working set of adapters kept resident in one AdapterLayer's pools.

    `host` maps an adapter key to (a_t_bits [r, d_in], b_bits [r, d_out], alpha)
    (bf16 tensors, host or device).  map_batch() turns the per-token keys of a
    batch into slot ids, loading the adapters that are not resident into the
    slots the LRU slot manager (lora_slot_cache_*) picks and pinning every slot
    the batch uses; release() unpins them once the batch has run.
    """

    def __init__(self, layer: AdapterLayer, host):
        self.layer = layer
        self.host = host
        self.slots = B.SlotCache(layer.S)

    def map_batch(self, keys, stream=None):
        """keys: per-token adapter keys (-1 = base model only).
        Returns (ids int32 tensor on the layer's device, pinned slot list)."""
        slot_of, pinned = {}, []
        for k in keys:
            k = int(k)
            if k < 0 or k in slot_of:
                continue
            slot, hit, evicted = self.slots.acquire(k, pin=True)
            pinned.append(slot)
            if not hit:
                if evicted >= 0:
                    self.layer.evict(slot, stream=stream)
                at, b, alpha = self.host[k]
                self.layer.load(slot, at.shape[0], alpha, at, b, stream=stream)
            slot_of[k] = slot
        ids = torch.tensor([slot_of.get(int(k), -1) for k in keys], dtype=torch.int32,
                           device=self.layer.device)
        return ids, pinned

    def release(self, pinned) -> None:
        for s in pinned:
            self.slots.unpin(s)


class PrefetchTicket:
    """A batch whose adapters are being brought in: its slot ids (host), the
    slots it pins and the event that marks the end of its loads."""

    def __init__(self, ids_host: torch.Tensor, pinned, ready: torch.cuda.Event, misses: int, bytes_loaded: int):
        self.ids_host, self.pinned, self.ready = ids_host, pinned, ready
        self.misses, self.bytes_loaded = misses, bytes_loaded


class AdapterPrefetcher:
    """Brings the adapters of upcoming batches into one AdapterLayer's pools on a
    copy stream while the current batch computes.

    Page "Multi-LoRA Serving in Production", section "Production Engineering
    Guidelines", "Asynchronous Prefetching and Request Queuing": on a cache
    miss the weights move from pinned host memory into the GPU pool with a
    non-blocking cudaMemcpyAsync, and the request waits an iteration or two
    until the transfer lands instead of stalling the batches already running.
    Page "LoRA Adapters at Serve Time with vLLM Multi-LoRA", section "The
    Inference Mechanism: A Worked Scenario", step "Eviction": the least
    recently used adapter makes room (lora_slot_cache_*, which never picks a
    slot pinned by a batch that has not been released).

    Ordering, all on the device (the host never waits):
      * a load into slot s first makes the copy stream wait for the event
        recorded after the last batch that read s, so pages are not
        overwritten under a batch still in flight; pages freed by an eviction
        are reused only by later loads on the same copy stream;
      * the compute stream waits for a ticket's `ready` event before the batch
        that uses it.
    `host` maps an adapter key to (a_t_bits [r, d_in], b_bits [r, d_out], alpha):
    pinned host tensors give asynchronous transfers.
    """

    def __init__(self, layer: AdapterLayer, host, copy_stream: Optional[torch.cuda.Stream] = None):
        self.layer = layer
        self.host = host
        self.slots = B.SlotCache(layer.S)
        self.copy = copy_stream or torch.cuda.Stream(device=layer.device)
        self.last_use = [None] * layer.S

    def prefetch(self, keys) -> PrefetchTicket:
        """Make every key of a coming batch resident (pinning its slot) and return
        its ticket; the loads of the misses are queued on the copy stream."""
        slot_of, pinned = {}, []
        misses, nbytes = 0, 0
        for k in keys:
            k = int(k)
            if k < 0 or k in slot_of:
                continue
            slot, hit, evicted = self.slots.acquire(k, pin=True)
            pinned.append(slot)
            if not hit:
                ev = self.last_use[slot]
                if ev is not None:
                    self.copy.wait_event(ev)
                if evicted >= 0:
                    self.layer.evict(slot, stream=self.copy)
                at, b, alpha = self.host[k]
                self.layer.load(slot, at.shape[0], alpha, at, b, stream=self.copy)
                misses += 1
                nbytes += at.numel() * at.element_size() + b.numel() * b.element_size()
            slot_of[k] = slot
        ready = torch.cuda.Event()
        ready.record(self.copy)
        ids = torch.tensor([slot_of.get(int(k), -1) for k in keys], dtype=torch.int32)
        return PrefetchTicket(ids, pinned, ready, misses, nbytes)

    def begin(self, ticket: PrefetchTicket, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Order `stream` (default: the current stream) after the ticket's loads and
        return the batch's slot ids on the device."""
        stream = stream or torch.cuda.current_stream(self.layer.device)
        stream.wait_event(ticket.ready)
        with torch.cuda.stream(stream):
            return ticket.ids_host.to(self.layer.device, non_blocking=True)

    def end(self, ticket: PrefetchTicket, stream: Optional[torch.cuda.Stream] = None) -> None:
        """After the batch's kernels are queued on `stream`: record when they finish
        reading its slots and release the pins."""
        stream = stream or torch.cuda.current_stream(self.layer.device)
        done = torch.cuda.Event()
        done.record(stream)
        for s in ticket.pinned:
            self.last_use[s] = done
            self.slots.unpin(s)
