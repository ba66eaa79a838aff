"""Seeded synthetic inputs for the heterogeneous-batch LoRA adapter branch.

This module only draws random data and arranges it; it holds none of the
method's arithmetic (no shrink, no expand, no scaling).  Both the oracle
tests and the CUDA path consume what it returns, so that the two sides see
bit-identical inputs.

Shapes follow the workloads of the pages:
  * "Multi-LoRA Serving in Production" (llms.blog), section "The Mathematical
    Anatomy of Heterogeneous Batches": row-vector layout X [T, d_in],
    A [d_in, r], B [r, d_out].
  * "Multi-LoRA Serving Architecture ... (2026)" (iotdigitaltwinplm.com),
    section "The memory arithmetic that makes it work": 7B/8B projection
    widths 4096 / 11008 / 14336; section "An adapter-cache LRU simulator":
    Zipf popularity p_i proportional to i^-s over i = 1..n.

Value recipe (all configs): X, A, B ~ N(0,1)/sqrt(fan_in) rounded to bf16 by
round-to-nearest-even (torch ``.to(bfloat16)``), fan_in = d_in for X and A and
r for B; Y_base ~ N(0,1) in fp32.  alpha: the tiny correctness case fixes
alpha = 2r; elsewhere the configs leave it open, and every slot draws its own
alpha from {r/2, 3r/2, 3r, 7, 2.9r} (fp32 values), so that neighbouring slots
carry different scales alpha/r and a kernel that reads another slot's scale
fails parity.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

PAGE_ROWS = 16
MAX_RANK = 64


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float data to the nearest bf16 value (RNE); return float32 holding it."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of float32 data that already holds bf16 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def zipf_weights(n: int, s: float) -> np.ndarray:
    """Normalised Zipf popularity, p_i proportional to i^-s for i = 1..n."""
    w = np.arange(1, n + 1, dtype=np.float64) ** (-float(s))
    return w / w.sum()


@dataclasses.dataclass
class Adapter:
    rank: int
    alpha: float
    A: np.ndarray  # [d_in, r] float32 holding bf16 values
    B: np.ndarray  # [r, d_out] float32 holding bf16 values


def draw_alphas(seed: int, ranks) -> np.ndarray:
    """One alpha per slot (fp32), drawn from {r/2, 3r/2, 3r, 7, 2.9r}; 0 for an empty slot."""
    r = np.asarray(ranks, dtype=np.int32)
    rf = r.astype(np.float32)
    table = np.stack([np.float32(0.5) * rf, np.float32(1.5) * rf, np.float32(3.0) * rf,
                      np.full_like(rf, np.float32(7.0)), np.float32(2.9) * rf]).astype(np.float32)
    pick = np.random.default_rng([seed, 7]).integers(0, table.shape[0], size=len(r))
    a = table[pick, np.arange(len(r))].astype(np.float32)
    a[r <= 0] = 0
    return a


class Adapters:
    """Per-slot adapters, each drawn from its own seed on first access, so a
    large resident pool never has to be held in host memory at once.
    alphas: fp32 alpha per slot (default: draw_alphas(seed, ranks))."""

    def __init__(self, seed: int, d_in: int, d_out: int, ranks: np.ndarray, cache: bool = True, alphas=None):
        self.seed, self.d_in, self.d_out = seed, d_in, d_out
        self.rank_of = np.asarray(ranks, dtype=np.int32)
        self.alpha_of = (draw_alphas(seed, self.rank_of) if alphas is None
                         else np.asarray(alphas, dtype=np.float32).copy())
        self._cache = {} if cache else None

    def __len__(self) -> int:
        return len(self.rank_of)

    def __getitem__(self, i: int) -> Optional[Adapter]:
        i = int(i)
        r = int(self.rank_of[i])
        if r <= 0:
            return None
        if self._cache is not None and i in self._cache:
            return self._cache[i]
        rng = np.random.default_rng([self.seed, 100, i])
        A = bf16_round(rng.standard_normal((self.d_in, r), dtype=np.float32) / np.float32(np.sqrt(self.d_in)))
        B = bf16_round(rng.standard_normal((r, self.d_out), dtype=np.float32) / np.float32(np.sqrt(r)))
        ad = Adapter(rank=r, alpha=float(self.alpha_of[i]), A=A, B=B)
        if self._cache is not None:
            self._cache[i] = ad
        return ad

    def __iter__(self):
        for i in range(len(self)):
            yield self[i]


@dataclasses.dataclass
class Workload:
    name: str
    d_in: int
    d_out: int
    X: np.ndarray          # [T, d_in] float32 (bf16 values)
    Y_base: np.ndarray     # [T, d_out] float32
    ids: np.ndarray        # [T] int32, -1 = base model only
    adapters: Adapters     # one entry per slot; None = empty slot
    page_ids: np.ndarray   # seeded physical page ids per slot: [S, 2, 4] (unused -1)
    pages_a: int           # pages in the d_in-wide pool
    pages_b: int           # pages in the d_out-wide pool

    @property
    def T(self) -> int:
        return int(self.X.shape[0])

    @property
    def S(self) -> int:
        return len(self.adapters)

    def ranks(self) -> np.ndarray:
        return self.adapters.rank_of.copy()

    def alphas(self) -> np.ndarray:
        return self.adapters.alpha_of.copy()

    def scales_f32(self) -> np.ndarray:
        """alpha/r per slot, one fp32 division (as the library's loader does it);
        both sides widen this value."""
        r = self.adapters.rank_of
        out = np.zeros(len(r), dtype=np.float32)
        nz = r > 0
        out[nz] = self.adapters.alpha_of[nz] / r[nz].astype(np.float32)
        return out

    def distinct(self) -> int:
        v = self.ids[(self.ids >= 0) & (self.ids < self.S)]
        return int(len(np.unique(v)))


def _assign_pages(seed: int, ranks: np.ndarray, extra_pages: int = 3):
    """Shuffled physical page ids for every (slot, matrix, page) of the resident adapters."""
    rng = np.random.default_rng([seed, 5])
    S = len(ranks)
    need = (np.maximum(ranks, 0).astype(np.int64) + PAGE_ROWS - 1) // PAGE_ROWS
    total = int(need.sum())
    pid = np.full((S, 2, 4), -1, dtype=np.int32)
    n_pool = total + extra_pages
    for m in range(2):
        order = rng.permutation(n_pool)[:total].astype(np.int32)
        k = 0
        for i in range(S):
            c = int(need[i])
            pid[i, m, :c] = order[k:k + c]
            k += c
    return pid, n_pool, n_pool


def _finish(name, seed, d_in, d_out, ids, ranks, alphas=None) -> Workload:
    T = len(ids)
    rx = np.random.default_rng([seed, 2])
    X = bf16_round(rx.standard_normal((T, d_in), dtype=np.float32) / np.float32(np.sqrt(d_in)))
    ry = np.random.default_rng([seed, 3])
    Y_base = ry.standard_normal((T, d_out), dtype=np.float32)
    ranks = np.asarray(ranks, dtype=np.int32)
    pid, na, nb = _assign_pages(seed, ranks)
    return Workload(name=name, d_in=d_in, d_out=d_out, X=X, Y_base=Y_base,
                    ids=np.ascontiguousarray(ids, dtype=np.int32),
                    adapters=Adapters(seed, d_in, d_out, ranks, cache=len(ranks) <= 256, alphas=alphas),
                    page_ids=pid, pages_a=na, pages_b=nb)


# ---------------------------------------------------------------------------
# The five workload shapes
# ---------------------------------------------------------------------------

def tiny(seed: int = 0) -> Workload:
    """d_in = d_out = 256, 8 decode tokens, 3 adapters of rank 4, 8, 16, uniform ids,
    alpha = 2r (the one config that fixes alpha)."""
    rng = np.random.default_rng([seed, 1])
    ids = rng.integers(0, 3, size=8)
    ranks = [4, 8, 16]
    return _finish("tiny_d256_T8", seed, 256, 256, ids, ranks, alphas=[2.0 * r for r in ranks])


def decode_q_proj_7b(seed: int = 1, T: int = 64) -> Workload:
    """d = 4096, one token per sequence, 32 resident rank-16 adapters drawn
    Zipf(1.0) without replacement from a 1000-adapter catalogue; each token draws
    a resident adapter with its renormalised Zipf weight."""
    rng = np.random.default_rng([seed, 1])
    w = zipf_weights(1000, 1.0)
    cat = rng.choice(1000, size=32, replace=False, p=w)
    p = w[cat] / w[cat].sum()
    ids = rng.choice(32, size=T, p=p)
    return _finish(f"decode_q_proj_7b_T{T}", seed, 4096, 4096, ids, [16] * 32)


def mixed_mlp(seed: int = 2, which: str = "up", T: int = 256) -> Workload:
    """256 decode tokens through the MLP up (4096 -> 11008) or down (11008 -> 4096)
    projection; 128 resident adapters with ranks uniform over {8,16,32,64};
    tokens assigned by Zipf(1.1) over the resident slots."""
    rng = np.random.default_rng([seed, 1])
    d_in, d_out = (4096, 11008) if which == "up" else (11008, 4096)
    ranks = rng.choice(np.array([8, 16, 32, 64]), size=128)
    slot_order = rng.permutation(128)
    ids = slot_order[rng.choice(128, size=T, p=zipf_weights(128, 1.1))]
    return _finish(f"mixed_mlp_{which}_T{T}", seed, d_in, d_out, ids, ranks)


def prefill(seed: int = 3, n_seq: int = 16, len_lo: int = 128, len_hi: int = 2048,
            d: int = 4096) -> Workload:
    """16 sequences of length uniform in [128, 2048], each one adapter; 6 distinct
    adapters with ranks drawn from {8,16,32,64}; tokens of a sequence are contiguous."""
    rng = np.random.default_rng([seed, 1])
    n_ad = 6
    ranks = rng.choice(np.array([8, 16, 32, 64]), size=n_ad)
    lens = rng.integers(len_lo, len_hi + 1, size=n_seq)
    seq_ad = rng.permutation(np.arange(n_seq) % n_ad)
    ids = np.concatenate([np.full(int(L), int(a)) for L, a in zip(lens, seq_ad)])
    return _finish(f"prefill_{n_seq}seq_T{len(ids)}", seed, d, d, ids, ranks)


def sweep_8b(seed: int = 4, T: int = 64, regime: str = "distinct", pool: int = 512,
             d_in: int = 4096, d_out: int = 14336, rank: int = 64) -> Workload:
    """d_in = 4096, d_out = 14336, rank 64, a pool of 512 resident adapters;
    regime "one": every token on one adapter; "distinct": token t uses
    perm[t mod 512] so min(T, 512) distinct adapters."""
    rng = np.random.default_rng([seed, 1])
    if regime == "one":
        ids = np.full(T, int(rng.integers(0, pool)))
    else:
        perm = rng.permutation(pool)
        ids = perm[np.arange(T) % pool]
    return _finish(f"sweep_8b_{regime}_T{T}", seed, d_in, d_out, ids, [rank] * pool)


def random_small(seed: int, T: int, d_in: int, d_out: int, S: int,
                 ranks=(1, 4, 8, 16), p_none: float = 0.1, p_empty: float = 0.0) -> Workload:
    """Random small case: mixed ranks, some id = -1 tokens, optional empty slots."""
    rng = np.random.default_rng([seed, 1])
    rk = rng.choice(np.array(ranks), size=S)
    rk[rng.random(S) < p_empty] = 0
    ids = rng.integers(0, S, size=T)
    ids[rng.random(T) < p_none] = -1
    return _finish(f"random_T{T}_{d_in}x{d_out}_S{S}", seed, d_in, d_out, ids, rk)


def segments(seed: int, lens, d_in: int, d_out: int, S: int, ranks=(1, 4, 8, 16, 33, 64),
             reuse: bool = False) -> Workload:
    """Prefill-like batch: sequence i brings lens[i] consecutive tokens that all use
    one adapter slot (distinct slots unless `reuse`, which lets sequences share a
    slot so that its tokens are no longer contiguous)."""
    rng = np.random.default_rng([seed, 1])
    rk = rng.choice(np.array(ranks), size=S)
    if reuse:
        seg_slot = rng.integers(0, S, size=len(lens))
    else:
        assert len(lens) <= S
        seg_slot = rng.permutation(S)[:len(lens)]
    ids = np.concatenate([np.full(int(L), int(a)) for L, a in zip(lens, seg_slot)]) if len(lens) else np.zeros(0)
    return _finish(f"segments_{len(lens)}_T{len(ids)}_{d_in}x{d_out}", seed, d_in, d_out, ids, rk)


def by_name(name: str, **kw) -> Workload:
    table = {
        "tiny": tiny,
        "decode_q_proj_7b": decode_q_proj_7b,
        "mixed_mlp_up": lambda **k: mixed_mlp(which="up", **k),
        "mixed_mlp_down": lambda **k: mixed_mlp(which="down", **k),
        "prefill": prefill,
        "sweep_8b_one": lambda **k: sweep_8b(regime="one", **k),
        "sweep_8b_distinct": lambda **k: sweep_8b(regime="distinct", **k),
    }
    return table[name](**kw)


def subset_for_tokens(wl: Workload, tokens) -> tuple:
    """(X, Y_base, ids, A list, B list, scales) restricted to `tokens`, with the
    slots they use renumbered 0..k-1 (to run the oracle on sampled outputs)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    ids = wl.ids[tokens]
    used = sorted({int(i) for i in ids if 0 <= i < wl.S and wl.adapters.rank_of[i] > 0})
    remap = {s: j for j, s in enumerate(used)}
    new_ids = np.array([remap.get(int(i), -1 if i == -1 else len(used) + 7) for i in ids], dtype=np.int32)
    A = [wl.adapters[s].A for s in used]
    Bm = [wl.adapters[s].B for s in used]
    sc = wl.scales_f32()[used] if used else np.zeros(0, np.float32)
    return wl.X[tokens], wl.Y_base[tokens], new_ids, A, Bm, sc


def shard_tokens(T: int, rank: int, world: int):
    """Contiguous token range [lo, hi) that data-parallel replica `rank` of `world` takes."""
    base, rem = divmod(T, world)
    lo = rank * base + min(rank, rem)
    hi = lo + base + (1 if rank < rem else 0)
    return lo, hi
