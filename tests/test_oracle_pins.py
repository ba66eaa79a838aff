"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

None of these checks re-types the oracle's own formula: each compares it with
a different route to the same number (a hand-worked example, the merged-weight
identity, a dense library matmul, a closed form, an invariant, a library sort,
or the pages' printed memory arithmetic).  The mutation tests at the end plant
plausible mistakes in copies of the oracle and show that some pin fails.
"""
import os

import numpy as np
import pytest

from oracle import lora_oracle as O
from oracle import build_oracle as OC
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def numpy_apply(X, Yb, ids, A, B, sc):
    return O.lora_apply(X, Yb, ids, A, B, sc)


def c_apply(X, Yb, ids, A, B, sc):
    return OC.lora_apply_c(X, Yb, ids, A, B, sc, nthreads=2)


def split_apply(X, Yb, ids, A, B, sc):
    """shrink followed by expand-add, the two-step form of the same method."""
    V, e1 = O.lora_shrink(X, ids, A)
    V = np.nan_to_num(V)
    Y, e2 = O.lora_expand_add(V, Yb, ids, B, sc)
    return Y, e1 | e2


IMPLS = {"numpy": numpy_apply, "c": c_apply, "split": split_apply}


# ---------------------------------------------------------------------------
# Pin checks, each taking an implementation of lora_apply
# ---------------------------------------------------------------------------

def _load_hand_example():
    rows = []
    with open(os.path.join(GOLDEN, "hand_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    rows = np.array(rows)
    ids = rows[:, 1].astype(np.int32)
    X = rows[:, 2:5].astype(np.float32)
    Yb = rows[:, 5:7].astype(np.float32)
    Yexp = rows[:, 7:9]
    A = [np.array([[1, 0], [0, 1], [2, 1]], np.float32), np.array([[1], [1], [1]], np.float32)]
    B = [np.array([[3, -1], [1, 2]], np.float32), np.array([[0.5, -2]], np.float32)]
    sc = np.array([4.0 / 2, 1.0 / 1], np.float32)
    return X, Yb, ids, A, B, sc, Yexp


def pin_hand_example(apply):
    X, Yb, ids, A, B, sc, Yexp = _load_hand_example()
    Y, err = apply(X, Yb, ids, A, B, sc)
    return err == 0 and np.array_equal(Y, Yexp)


def _rand_case(seed, T=7, d_in=12, d_out=10, ranks=(1, 3, 5, 8)):
    rng = np.random.default_rng(seed)
    A = [W.bf16_round(rng.standard_normal((d_in, r)).astype(np.float32)) for r in ranks]
    B = [W.bf16_round(rng.standard_normal((r, d_out)).astype(np.float32)) for r in ranks]
    sc = (rng.integers(1, 9, size=len(ranks)) / np.array(ranks)).astype(np.float32)
    X = W.bf16_round(rng.standard_normal((T, d_in)).astype(np.float32))
    Yb = rng.standard_normal((T, d_out)).astype(np.float32)
    ids = rng.integers(0, len(ranks), size=T).astype(np.int32)
    return X, Yb, ids, A, B, sc


def pin_merge_identity(apply, seed=11):
    """Unmerged output == X (W0 + s A B) for every token's adapter (pre-merge identity,
    llms.blog "The Mathematical Anatomy ..."; iotdigitaltwinplm "Why merging per tenant
    does not scale").  d_in != d_out, so a transposed operand cannot pass."""
    X, _, ids, A, B, sc = _rand_case(seed)
    rng = np.random.default_rng(seed + 1)
    W0 = rng.standard_normal((X.shape[1], B[0].shape[1]))
    Yb = X.astype(np.float64) @ W0
    Y, err = apply(X, Yb.astype(np.float32), ids, A, B, sc)
    Yb32 = Yb.astype(np.float32).astype(np.float64)
    ok = err == 0
    for t in range(X.shape[0]):
        i = ids[t]
        Wm = O.merged_weight(W0, A[i], B[i], sc[i])
        ref = X[t].astype(np.float64) @ Wm - (X[t].astype(np.float64) @ W0) + Yb32[t]
        ok &= np.allclose(Y[t], ref, rtol=1e-12, atol=1e-12)
    return bool(ok)


def pin_one_adapter_dense(apply, seed=12):
    """All tokens on one adapter == one dense product Y_base + s (X A) B
    (iotdigitaltwinplm "Heterogeneous batching": one adapter is read once)."""
    X, Yb, _, A, B, sc = _rand_case(seed, T=9)
    ids = np.full(X.shape[0], 2, np.int32)
    Y, err = apply(X, Yb, ids, A, B, sc)
    ref = Yb.astype(np.float64) + np.float64(sc[2]) * np.matmul(
        np.matmul(X.astype(np.float64), A[2].astype(np.float64)), B[2].astype(np.float64))
    return err == 0 and np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


def pin_zero_b(apply, seed=13):
    """B = 0 gives Delta W = A B = 0, so Y == Y_base exactly."""
    X, Yb, ids, A, B, sc = _rand_case(seed)
    B0 = [np.zeros_like(b) for b in B]
    Y, err = apply(X, Yb, ids, A, B0, sc)
    return err == 0 and np.array_equal(Y, Yb.astype(np.float64))


def pin_selector(apply, seed=14):
    """A = [I_r; 0], B = [I_r 0]  =>  Delta Y[t, :r] = s X[t, :r], zero elsewhere."""
    rng = np.random.default_rng(seed)
    d_in, d_out, T = 11, 9, 6
    ranks = (2, 5)
    A = [np.eye(d_in, r, dtype=np.float32) for r in ranks]
    B = [np.eye(r, d_out, dtype=np.float32) for r in ranks]
    sc = np.array([1.5, 0.25], np.float32)
    X = W.bf16_round(rng.standard_normal((T, d_in)).astype(np.float32))
    Yb = np.zeros((T, d_out), np.float32)
    ids = np.array([0, 1, 1, 0, 1, 0], np.int32)
    Y, err = apply(X, Yb, ids, A, B, sc)
    ok = err == 0
    for t in range(T):
        r = ranks[ids[t]]
        exp = np.zeros(d_out)
        exp[:r] = np.float64(sc[ids[t]]) * X[t, :r].astype(np.float64)
        ok &= np.array_equal(Y[t], exp)
    return bool(ok)


def pin_rank1(apply, seed=15):
    """r = 1: Delta Y[t, c] = s (x_t . a) b_c."""
    rng = np.random.default_rng(seed)
    d_in, d_out, T = 8, 6, 4
    a = np.arange(1, d_in + 1, dtype=np.float32).reshape(d_in, 1)
    b = np.array([[1, -2, 0.5, 3, 0, -1]], np.float32)
    X = rng.integers(-3, 4, size=(T, d_in)).astype(np.float32)
    Yb = np.zeros((T, d_out), np.float32)
    ids = np.zeros(T, np.int32)
    sc = np.array([0.5], np.float32)
    Y, err = apply(X, Yb, ids, [a], [b], sc)
    dots = X.astype(np.float64) @ np.arange(1, d_in + 1, dtype=np.float64)
    exp = 0.5 * dots[:, None] * b.astype(np.float64)
    return err == 0 and np.array_equal(Y, exp)


def pin_permutation(apply, seed=16):
    """Each token sees only its own adapter (iotdigitaltwinplm "Trade-offs, Gotchas"):
    permuting the batch permutes the output rows, bit for bit."""
    X, Yb, ids, A, B, sc = _rand_case(seed, T=10)
    P = np.random.default_rng(seed).permutation(X.shape[0])
    Y1, e1 = apply(X, Yb, ids, A, B, sc)
    Y2, e2 = apply(X[P], Yb[P], ids[P], A, B, sc)
    return e1 == 0 and e2 == 0 and np.array_equal(Y1[P], Y2)


def pin_ids_none_and_invalid(apply, seed=17):
    """id = -1 rows keep Y_base; an id outside [-1, S) keeps Y_base and raises bit 1;
    the other rows are those of the clean batch."""
    X, Yb, ids, A, B, sc = _rand_case(seed, T=8)
    Yc, _ = apply(X, Yb, ids, A, B, sc)
    ids2 = ids.copy()
    ids2[1] = -1
    ids2[4] = len(A)      # out of range
    ids2[6] = -5          # out of range
    Y, err = apply(X, Yb, ids2, A, B, sc)
    ok = err == O.ERR_BAD_ID
    for t in (1, 4, 6):
        ok &= np.array_equal(Y[t], Yb[t].astype(np.float64))
    for t in (0, 2, 3, 5, 7):
        ok &= np.array_equal(Y[t], Yc[t])
    return bool(ok)


def pin_scale_linear(apply, seed=18):
    """Delta Y is linear in s: doubling s doubles Delta Y exactly (powers of two)."""
    X, _, ids, A, B, sc = _rand_case(seed)
    Yb = np.zeros((X.shape[0], B[0].shape[1]), np.float32)
    Y1, _ = apply(X, Yb, ids, A, B, sc)
    Y2, _ = apply(X, Yb, ids, A, B, (2 * sc).astype(np.float32))
    return np.array_equal(2 * Y1, Y2) and np.abs(Y1).max() > 0


PINS = [pin_hand_example, pin_merge_identity, pin_one_adapter_dense, pin_zero_b,
        pin_selector, pin_rank1, pin_permutation, pin_ids_none_and_invalid, pin_scale_linear]


@pytest.mark.parametrize("impl", sorted(IMPLS))
@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(impl, pin):
    assert pin(IMPLS[impl])


def test_merged_weight_selector_closed_form():
    """merged_weight(W0, [I_r; 0], [I_r 0], s) = W0 + s E_r, with E_r the identity on
    the leading r x r block and zero elsewhere (d_in != d_out, s not 1)."""
    rng = np.random.default_rng(31)
    d_in, d_out, r, s = 11, 9, 4, np.float32(0.375)
    W0 = rng.standard_normal((d_in, d_out))
    A = np.zeros((d_in, r), np.float32)
    A[:r, :r] = np.eye(r)
    B = np.zeros((r, d_out), np.float32)
    B[:r, :r] = np.eye(r)
    E = np.zeros((d_in, d_out))
    E[:r, :r] = np.eye(r)
    assert np.array_equal(O.merged_weight(W0, A, B, s), W0 + 0.375 * E)


def test_merged_weight_rank1_closed_form():
    """A rank-1 adapter a b^T merges to W0 + s a b^T, element by element."""
    rng = np.random.default_rng(32)
    a = W.bf16_round(rng.standard_normal((7, 1)).astype(np.float32))
    b = W.bf16_round(rng.standard_normal((1, 5)).astype(np.float32))
    W0 = rng.standard_normal((7, 5))
    s = np.float32(1.25)
    got = O.merged_weight(W0, a, b, s)
    for j in range(7):
        for c in range(5):
            assert got[j, c] == W0[j, c] + 1.25 * (float(a[j, 0]) * float(b[0, c]))


def test_c_and_numpy_oracles_agree_on_generated_workload():
    wl = W.random_small(seed=5, T=40, d_in=64, d_out=48, S=6, ranks=(1, 4, 8, 16, 33, 64))
    A = [a.A for a in wl.adapters]
    B = [a.B for a in wl.adapters]
    Y1, e1 = O.lora_apply(wl.X, wl.Y_base, wl.ids, A, B, wl.scales_f32())
    Y2, e2 = OC.lora_apply_c(wl.X, wl.Y_base, wl.ids, A, B, wl.scales_f32(), nthreads=3)
    assert e1 == e2
    np.testing.assert_allclose(Y1, Y2, rtol=1e-13, atol=1e-13)


def test_empty_slot_sets_bit_and_keeps_row():
    X, Yb, ids, A, B, sc = _rand_case(19, T=6)
    A2, B2 = list(A), list(B)
    A2[1] = None
    B2[1] = None
    ids = np.array([0, 1, 2, 1, 3, 0], np.int32)
    for impl in IMPLS.values():
        Y, err = impl(X, Yb, ids, A2, B2, sc)
        assert err == O.ERR_EMPTY_SLOT
        assert np.array_equal(Y[1], Yb[1].astype(np.float64))
        assert np.array_equal(Y[3], Yb[3].astype(np.float64))


# ---------------------------------------------------------------------------
# Plan (grouping by adapter), paging and memory arithmetic
# ---------------------------------------------------------------------------

def test_segment_plan_matches_library_stable_sort():
    rng = np.random.default_rng(21)
    for trial in range(20):
        S = int(rng.integers(1, 40))
        T = int(rng.integers(0, 300))
        ranks = rng.integers(0, 3, size=S) * 16  # some empty slots
        ids = rng.integers(-2, S + 2, size=T)
        perm, seg, err = O.segment_plan(ids, ranks)
        valid = np.array([(0 <= i < S) and ranks[i] > 0 for i in ids], dtype=bool)
        tok = np.nonzero(valid)[0]
        ref = tok[np.argsort(ids[tok], kind="stable")]
        assert np.array_equal(perm, ref)
        counts = np.bincount(ids[tok], minlength=S)
        assert np.array_equal(seg, np.concatenate([[0], np.cumsum(counts)]))
        bad = ((ids < -1) | (ids >= S)).any()
        empty = any((0 <= i < S) and ranks[i] == 0 for i in ids)
        assert err == (O.ERR_BAD_ID if bad else 0) | (O.ERR_EMPTY_SLOT if empty else 0)


def test_page_row_hand_values():
    # page table row [7, 2, 9]: rank-rows 0..15 in page 7, 16..31 in page 2, 32.. in page 9
    pt = [7, 2, 9, -1]
    assert O.page_row(pt, 0) == 112
    assert O.page_row(pt, 15) == 127
    assert O.page_row(pt, 16) == 32
    assert O.page_row(pt, 17) == 33
    assert O.page_row(pt, 40) == 9 * 16 + 8


def test_page_gather_round_trip_shuffled():
    rng = np.random.default_rng(22)
    width, n_pages = 24, 9
    pool = np.full((n_pages * 16, width), np.nan)
    for r in (1, 4, 15, 16, 17, 40, 64):
        mat = rng.standard_normal((r, width))
        pages = rng.permutation(n_pages)[: (r + 15) // 16]
        for k in range(r):
            pool[O.page_row(pages, k)] = mat[k]
        back = O.gather_rows(pool, pages, r)
        assert np.array_equal(back, mat)


def _golden_memory():
    out = {}
    with open(os.path.join(GOLDEN, "adapter_memory_arithmetic.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v, tol = line.split()[:3]
                out[k] = (float(v), float(tol))
    return out


def test_adapter_params_match_printed_arithmetic():
    g = _golden_memory()
    h, kv, mlp, L = 4096, 1024, 14336, 32
    allp = [(h, h), (h, kv), (h, kv), (h, h), (h, mlp), (h, mlp), (mlp, h)]
    attn = allp[:4]

    def check(key, val):
        ref, tol = g[key]
        assert abs(val - ref) <= tol * ref, (key, val, ref)

    check("params_per_unit_rank_per_layer", O.adapter_params(1, allp))
    check("params_per_layer_r16", O.adapter_params(16, allp))
    check("params_32_layers_r16", L * O.adapter_params(16, allp))
    check("bytes_16bit_r16", 2 * L * O.adapter_params(16, allp))
    check("bytes_16bit_r64", 2 * L * O.adapter_params(64, allp))
    check("params_attention_only_r16", L * O.adapter_params(16, attn))
    check("bytes_attention_only_r16", 2 * L * O.adapter_params(16, attn))
    check("slot_bytes_32_slots_r64", 32 * 2 * L * O.adapter_params(64, allp))
    check("slot_bytes_32_slots_r8", 32 * 2 * L * O.adapter_params(8, allp))


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle must fail at least one pin
# ---------------------------------------------------------------------------

def _mutant(kind):
    def apply(X, Yb, ids, A, B, sc):
        X = np.asarray(X)
        T = X.shape[0]
        S = len(A)
        Y = np.array(Yb, dtype=np.float64, copy=True)
        err = 0
        for t in range(T):
            i = int(ids[t])
            if i == -1:
                continue
            if i < -1 or i >= S or A[i] is None:
                err |= O.ERR_BAD_ID if (i < -1 or i >= S) else O.ERR_EMPTY_SLOT
                continue
            x = X[t].astype(np.float64)
            a = A[i].astype(np.float64)
            b = B[i].astype(np.float64)
            s = np.float64(sc[i])
            if kind == "no_scale":
                s = 1.0
            if kind == "scale_times_r":
                s = s * a.shape[1]
            if kind == "sign":
                s = -s
            if kind == "drop_last_rank":
                a, b = a[:, :-1], b[:-1]
            if kind == "rank_shift" and a.shape[1] > 1:
                a = np.roll(a, 1, axis=1)
            if kind == "reversed_x":
                x = x[::-1]
            if kind == "neighbour_adapter":
                j = (i + 1) % S
                a, b = A[j].astype(np.float64), B[j].astype(np.float64)
            if kind == "skip_ybase":
                Y[t] = 0.0
            if kind == "first_token_adapter":
                j = int(ids[0]) if int(ids[0]) >= 0 else i
                a, b = A[j].astype(np.float64), B[j].astype(np.float64)
            if kind == "neighbour_scale":
                s = np.float64(sc[(i + 1) % S])
            Y[t] += s * ((x @ a) @ b)
        return Y, err
    return apply


MUTANTS = ["no_scale", "scale_times_r", "sign", "drop_last_rank", "rank_shift",
           "reversed_x", "neighbour_adapter", "skip_ybase", "first_token_adapter", "neighbour_scale"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_is_caught(kind):
    m = _mutant(kind)
    failed = []
    for pin in PINS:
        try:
            ok = pin(m)
        except Exception:
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"mutant {kind} passed every pin"
