"""Tensor-parallel adapter branch over Megatron-style sharded layers.

Page "Multi-LoRA Serving in Production" (llms.blog), sections "Distributed
Multi-LoRA: Tensor Parallelism Strategies", "Partitioning Rules for Linear
Layers" and "S-LoRA TP Communication Optimization":

* column-parallel layer (q/k/v, MLP gate/up): the base weight is split by
  output columns; A is replicated and B split by columns, so rank k computes
  x A B_k into its own output block with no communication;
* row-parallel layer (attention output, MLP down): the base weight is split by
  input rows; A is split by rows and B replicated, so rank k adds
  (x_k A_k) B to its partial base output and the layer's single all-reduce
  sums base and adapter partials together;
* the S-LoRA variant of the row-parallel layer for small ranks: B is split by
  columns as well, the rank-r partial vectors v_k = x_k A_k are summed across
  ranks (an all-reduce of a [T, r] tensor), and rank k adds s v B_k into its
  own column block of the partial output before the layer's all-reduce.

Every compute step runs in liblora (lora_apply, lora_shrink,
lora_expand_add_strided); the collectives go through torch.distributed (NCCL
on GPUs).  The `ops` argument of the classes below names the compute entry
points and defaults to the library; a test may pass a host implementation to
check the collective schedule on CPU ranks.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _binding as B
from .layer import AdapterLayer

COLUMN, ROW, ROW_V_EXCHANGE = "column", "row", "row_v_exchange"


def shard_range(n: int, rank: int, world: int, align: int = 8):
    """Contiguous block [lo, hi) of n columns (or rows) that `rank` of `world` holds;
    blocks are whole multiples of `align` except the last one."""
    if n % align:
        raise ValueError(f"width {n} is not a multiple of {align}")
    groups = n // align
    base, rem = divmod(groups, world)
    lo = rank * base + min(rank, rem)
    hi = lo + base + (1 if rank < rem else 0)
    return lo * align, hi * align


def shard_adapter(mode: str, A_t: torch.Tensor, Bm: torch.Tensor, rank: int, world: int):
    """(A^T shard, B shard) of one adapter for `rank`: A_t is [r, d_in], Bm [r, d_out]."""
    d_in, d_out = A_t.shape[1], Bm.shape[1]
    if mode == COLUMN:
        lo, hi = shard_range(d_out, rank, world)
        return A_t, Bm[:, lo:hi]
    ilo, ihi = shard_range(d_in, rank, world)
    if mode == ROW:
        return A_t[:, ilo:ihi], Bm
    if mode == ROW_V_EXCHANGE:
        olo, ohi = shard_range(d_out, rank, world)
        return A_t[:, ilo:ihi], Bm[:, olo:ohi]
    raise ValueError(mode)


class LibraryOps:
    """The library's compute entry points used by the tensor-parallel schedule."""

    @staticmethod
    def apply(layer: AdapterLayer, X, Y, ids, stream=None):
        layer.apply(X, Y, ids, stream=stream)

    @staticmethod
    def shrink(layer: AdapterLayer, X, ids, V, stream=None):
        layer.shrink(X, ids, V, stream=stream)

    @staticmethod
    def expand_add_block(layer: AdapterLayer, V, Y, col0: int, ids, stream=None):
        """Y[:, col0:col0 + layer.d_out] += s v B_k (Y row-major, rows Y.shape[1] apart)."""
        blk = Y[:, col0:col0 + layer.d_out]
        B.lora_expand_add_strided(V, blk, Y.shape[1], V.shape[0], layer.d_out, ids, layer.S, layer.ranks,
                                  layer.scales, layer.page_table, layer.pool_b, layer.ws, layer.err, stream)


class TPLoRA:
    """One rank's shard of an adapted linear layer under tensor parallelism.

    mode: COLUMN, ROW or ROW_V_EXCHANGE.  The rank's AdapterLayer holds pools of
    the shard's widths (A^T rows of width d_in or d_in/world, B rows of width
    d_out or d_out/world); load() takes the full adapter and keeps this rank's
    shard.
    """

    def __init__(self, mode: str, d_in: int, d_out: int, num_slots: int, pages: int, max_tokens: int,
                 rank: int, world: int, group=None, device="cuda", ops=None, layer=None):
        self.mode, self.rank, self.world, self.group = mode, rank, world, group
        self.d_in, self.d_out = d_in, d_out
        self.in_lo, self.in_hi = (0, d_in) if mode == COLUMN else shard_range(d_in, rank, world)
        self.out_lo, self.out_hi = (0, d_out) if mode == ROW else shard_range(d_out, rank, world)
        self.ops = ops or LibraryOps
        # `layer` (with `ops`) lets a test supply a host stand-in for the device state
        self.layer = layer if layer is not None else AdapterLayer(
            self.in_hi - self.in_lo, self.out_hi - self.out_lo, num_slots, pages, pages, max_tokens, device=device)

    def load(self, slot: int, rank: int, alpha: float, A_t: torch.Tensor, Bm: torch.Tensor,
             page_ids: Optional[torch.Tensor] = None, stream=None) -> None:
        a_t, b = shard_adapter(self.mode, A_t, Bm, self.rank, self.world)
        self.layer.load(slot, rank, alpha, a_t.contiguous(), b.contiguous(), page_ids=page_ids, stream=stream)

    def evict(self, slot: int, stream=None) -> None:
        self.layer.evict(slot, stream=stream)

    # -- the schedule, split into its local steps (a single-device test runs the
    #    ranks' steps in turn and stands in for the collectives) --

    def local_apply(self, X_local, Y_local, ids, stream=None) -> None:
        """COLUMN: Y_local [T, d_out/world] += s (X A) B_k.  ROW: Y_partial [T, d_out]
        += s (X_k A_k) B, X_local = X[:, in_lo:in_hi]."""
        assert self.mode in (COLUMN, ROW)
        self.ops.apply(self.layer, X_local, Y_local, ids, stream)

    def local_shrink(self, X_local, ids, V, stream=None) -> None:
        """ROW_V_EXCHANGE: V [T, 64] (zeroed by the caller) = x_k A_k, this rank's partial v."""
        assert self.mode == ROW_V_EXCHANGE
        self.ops.shrink(self.layer, X_local, ids, V, stream)

    def local_expand(self, V_sum, Y_partial, ids, stream=None) -> None:
        """ROW_V_EXCHANGE: Y_partial[:, out_lo:out_hi] += s v B_k with v summed over ranks."""
        assert self.mode == ROW_V_EXCHANGE
        self.ops.expand_add_block(self.layer, V_sum, Y_partial, self.out_lo, ids, stream)

    # -- the whole schedule with its collectives --

    def forward(self, X_local, Y, ids, reduce_output: bool = True, stream=None) -> None:
        """Run this rank's part of the layer.

        COLUMN: Y is the rank's output block; no communication.
        ROW / ROW_V_EXCHANGE: Y is the rank's partial output X_k W0_k (full width);
        the adapter's share is added and, with reduce_output, Y is all-reduced
        (the base layer's own all-reduce, now carrying base + adapter partials).
        """
        import torch.distributed as dist
        if self.mode == COLUMN:
            self.local_apply(X_local, Y, ids, stream)
            return
        if self.mode == ROW:
            self.local_apply(X_local, Y, ids, stream)
        else:
            V = torch.zeros((X_local.shape[0], B.MAX_RANK), dtype=Y.dtype, device=Y.device)
            self.local_shrink(X_local, ids, V, stream)
            dist.all_reduce(V, group=self.group)          # sum of the rank-r partials
            self.local_expand(V, Y, ids, stream)
        if reduce_output:
            dist.all_reduce(Y, group=self.group)
