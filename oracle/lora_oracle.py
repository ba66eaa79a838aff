"""fp64 CPU oracle of the heterogeneous-batch LoRA adapter branch.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
link this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, tables or helpers).

Every function is the plain definition written out, in float64, on the same
bf16-rounded inputs the GPU path receives.  Sources (page title, section):

* "Multi-LoRA Serving in Production" (llms.blog), "The Mathematical Anatomy of
  Heterogeneous Batches", eq. Y = X W0 + (alpha/r)(X A) B with A in
  R^{d_in x r}, B in R^{r x d_out}; each sequence i in the batch uses its own
  (A_i, B_i, r_i).
* same page, "Segmented Gather Matrix-Vector Multiplication (SGMV)": the shrink
  v_i = x_i A_i, then the expand v_i B_i scaled by alpha_i/r_i and added to the
  base output; requests are grouped by adapter.
* same page, "Unified Paging Architecture": adapter weights are sliced into
  pages along the rank dimension; a page table maps logical to physical pages.
* "Multi-LoRA Serving Architecture ... (2026)" (iotdigitaltwinplm.com),
  "Trade-offs, Gotchas, and What Goes Wrong": each token sees only its own
  adapter; base-model requests share the server (id = -1 below).
* same page, "The memory arithmetic that makes it work": an adapter on a
  projection costs r*(d_in + d_out) parameters.

Readings where the pages are silent:
  * orientation follows the llms.blog page (row vectors); the column-vector
    form on the iotdigitaltwinplm page is its transpose;
  * the scale alpha/r is part of the method (the ashishsrivastav page drops
    it, which is the special case alpha = r); it is handed over as one fp32
    value per slot and widened to fp64 here;
  * the scale multiplies the expanded sum: y += s * (v B);
  * an id outside [-1, S) or an id naming an empty slot (rank 0) leaves the row
    unchanged and raises an error bit; id = -1 means base model only.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, the merge identity, a library-routine special case, invariants,
a hand-computed golden example and the pages' printed memory arithmetic).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

ERR_BAD_ID = 1       # id < -1 or id >= S
ERR_EMPTY_SLOT = 2   # id names a slot that holds no adapter (rank 0)


def _check_id(i: int, S: int, ranks: Sequence[int]) -> int:
    if i == -1:
        return -1
    if i < -1 or i >= S:
        return ERR_BAD_ID
    if int(ranks[i]) <= 0:
        return ERR_EMPTY_SLOT
    return 0


def lora_apply(X, Y_base, ids, A: Sequence[Optional[np.ndarray]], B: Sequence[Optional[np.ndarray]],
               scales, ranks=None):
    """Y[t] = Y_base[t] + s_i * (X[t] A_i) B_i with i = ids[t]   (fp64).

    X      [T, d_in]   bf16-valued floats
    Y_base [T, d_out]  fp32
    ids    [T]         int, -1 = no adapter
    A[i]   [d_in, r_i], B[i] [r_i, d_out]  (None for an empty slot)
    scales [S]         fp32 alpha_i / r_i
    Returns (Y fp64 [T, d_out], error bits int).
    """
    X = np.asarray(X)
    T = X.shape[0]
    S = len(A)
    if ranks is None:
        ranks = [0 if a is None else a.shape[1] for a in A]
    Y = np.array(Y_base, dtype=np.float64, copy=True)
    err = 0
    for t in range(T):
        i = int(ids[t])
        e = _check_id(i, S, ranks)
        if e == -1:
            continue
        if e:
            err |= e
            continue
        x = X[t].astype(np.float64)
        v = x @ A[i].astype(np.float64)                       # shrink: rank-r_i vector
        Y[t] += np.float64(np.float32(scales[i])) * (v @ B[i].astype(np.float64))  # expand-add
    return Y, err


def lora_shrink(X, ids, A, ranks=None, max_rank: int = 64):
    """V[t, k] = sum_j X[t, j] A_i[j, k] for k < r_i  (fp64).

    Columns k >= r_i, and rows of tokens with no valid adapter, are NaN: the
    library leaves them untouched, so only the defined entries are compared.
    """
    X = np.asarray(X)
    T = X.shape[0]
    S = len(A)
    if ranks is None:
        ranks = [0 if a is None else a.shape[1] for a in A]
    V = np.full((T, max_rank), np.nan)
    err = 0
    for t in range(T):
        i = int(ids[t])
        e = _check_id(i, S, ranks)
        if e == -1:
            continue
        if e:
            err |= e
            continue
        r = A[i].shape[1]
        V[t, :r] = X[t].astype(np.float64) @ A[i].astype(np.float64)
    return V, err


def lora_expand_add(V, Y_base, ids, B, scales, ranks=None):
    """Y[t] = Y_base[t] + s_i * sum_k V[t, k] B_i[k, :] over k < r_i  (fp64)."""
    V = np.asarray(V)
    T = V.shape[0]
    S = len(B)
    if ranks is None:
        ranks = [0 if b is None else b.shape[0] for b in B]
    Y = np.array(Y_base, dtype=np.float64, copy=True)
    err = 0
    for t in range(T):
        i = int(ids[t])
        e = _check_id(i, S, ranks)
        if e == -1:
            continue
        if e:
            err |= e
            continue
        r = B[i].shape[0]
        Y[t] += np.float64(np.float32(scales[i])) * (V[t, :r].astype(np.float64) @ B[i].astype(np.float64))
    return Y, err


def merged_weight(W0, A, B, scale):
    """W' = W0 + s * A B, the single-tenant pre-merged matrix (fp64).

    "Multi-LoRA Serving in Production", "The Mathematical Anatomy of
    Heterogeneous Batches": merging folds the low-rank product into the base
    weight; the unmerged branch must give X W' for every token."""
    return np.asarray(W0, np.float64) + np.float64(np.float32(scale)) * (
        np.asarray(A, np.float64) @ np.asarray(B, np.float64))


def segment_plan(ids, ranks):
    """Group tokens by adapter slot (the SGMV grouping step), stably.

    Returns (perm, seg_start, err):
      perm       tokens with a valid adapter, ordered by slot ascending and,
                 within a slot, by original token index;
      seg_start  [S+1] with tokens of slot i at perm[seg_start[i]:seg_start[i+1]];
      err        error bits of the dropped invalid ids.
    Tokens with id = -1 are dropped silently.
    """
    ids = np.asarray(ids)
    S = len(ranks)
    buckets = [[] for _ in range(S)]
    err = 0
    for t in range(len(ids)):                       # one pass in token order = stable
        i = int(ids[t])
        e = _check_id(i, S, ranks)
        if e == -1:
            continue
        if e:
            err |= e
            continue
        buckets[i].append(t)
    seg_start = np.zeros(S + 1, dtype=np.int64)
    perm = []
    for i in range(S):
        seg_start[i] = len(perm)
        perm.extend(buckets[i])
    seg_start[S] = len(perm)
    return np.array(perm, dtype=np.int64), seg_start, err


def page_row(page_table_row, k: int, page_rows: int = 16) -> int:
    """Physical pool row holding logical rank-row k of one matrix of one slot:
    the page table names the physical page, the row offset inside it is k mod page_rows."""
    return int(page_table_row[k // page_rows]) * page_rows + (k % page_rows)


def gather_rows(pool_rows: np.ndarray, page_table_row, r: int, page_rows: int = 16) -> np.ndarray:
    """Logical [r, width] matrix read back from a paged pool through its page-table row."""
    return np.stack([pool_rows[page_row(page_table_row, k, page_rows)] for k in range(r)])


def adapter_params(rank: int, projections: Sequence[tuple]) -> int:
    """Parameters of one adapter: r * (d_in + d_out) summed over the projections."""
    return int(sum(int(rank) * (int(di) + int(do)) for di, do in projections))
