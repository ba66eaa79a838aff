"""The pool's slot manager (lora_slot_cache_*): exact LRU over the slots that
no running batch pins.

Pinned against the page "Multi-LoRA Serving Architecture ... (2026)", section
"An adapter-cache LRU simulator" (the hit rates it reports for Zipf streams,
tests/golden/lru_hit_rates.txt), and bit-exactly against a brute-force model of
LRU with pins on random operation sequences.  Host-only: no GPU is touched.
"""
import os

import numpy as np
import pytest

import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def B():
    from heterogeneous_adapter_batching_b200 import _binding as B
    B.load_library()
    return B


def _golden():
    rows = []
    for line in open(os.path.join(HERE, "golden", "lru_hit_rates.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            s, slots, pct = line.split()
            rows.append((float(s), int(slots), float(pct)))
    return rows


@pytest.mark.parametrize("s,slots,pct", _golden())
def test_hit_rate_matches_the_page(B, s, slots, pct):
    """500 adapters, 200,000 i.i.d. Zipf(s) requests: the LRU hit rate converges
    to a value the page reports rounded to whole percent; our stream is a
    different seeded draw of the same distribution."""
    rng = np.random.default_rng([7, int(s * 10), slots])
    req = rng.choice(500, size=200_000, p=W.zipf_weights(500, s))
    c = B.SlotCache(slots)
    hits = 0
    for a in req.tolist():
        hits += c.acquire(a)[1]
    h, m, e = c.stats()
    assert h == hits and h + m == len(req) and e == m - slots
    assert abs(100.0 * hits / len(req) - pct) <= 1.5


class Model:
    """Brute force: residents in recency order (least recent first)."""

    def __init__(self, n):
        self.key = [-1] * n
        self.pins = [0] * n
        self.order = []                       # resident slots, least recent first
        self.empty = list(range(n - 1, -1, -1))   # pop() gives the next empty slot

    def acquire(self, key, pin):
        if key in self.key:
            s = self.key.index(key)
            self.order.remove(s)
            hit, ev = True, -1
        else:
            if self.empty:
                s, ev = self.empty.pop(), -1
            else:
                free = [x for x in self.order if self.pins[x] == 0]
                if not free:
                    return "ALL_PINNED"
                s = free[0]
                self.order.remove(s)
                ev = self.key[s]
            self.key[s] = key
            hit = False
        self.order.append(s)
        if pin:
            self.pins[s] += 1
        return s, hit, ev

    def unpin(self, s):
        if self.pins[s] <= 0:
            return "INVALID"
        self.pins[s] -= 1
        return None

    def invalidate(self, s):
        if self.key[s] < 0:
            return None
        if self.pins[s] > 0:
            return "ALL_PINNED"
        self.order.remove(s)
        self.key[s] = -1
        self.empty.append(s)
        return None


@pytest.mark.parametrize("seed,n,keys", [(0, 1, 3), (1, 4, 10), (2, 16, 40), (3, 64, 200), (4, 7, 7)])
def test_matches_brute_force_model(B, seed, n, keys):
    rng = np.random.default_rng([seed, 77])
    c, m = B.SlotCache(n), Model(n)
    for _ in range(4000):
        op = rng.random()
        if op < 0.7:
            key, pin = int(rng.integers(0, keys)), bool(rng.random() < 0.3)
            want = m.acquire(key, pin)
            if want == "ALL_PINNED":
                with pytest.raises(B.LoraError) as ei:
                    c.acquire(key, pin)
                assert ei.value.rc == -9
            else:
                assert c.acquire(key, pin) == want
        elif op < 0.9:
            s = int(rng.integers(0, n))
            want = m.unpin(s)
            if want == "INVALID":
                with pytest.raises(B.LoraError) as ei:
                    c.unpin(s)
                assert ei.value.rc == -1
            else:
                c.unpin(s)
        else:
            s = int(rng.integers(0, n))
            want = m.invalidate(s)
            if want == "ALL_PINNED":
                with pytest.raises(B.LoraError) as ei:
                    c.invalidate(s)
                assert ei.value.rc == -9
            else:
                c.invalidate(s)
        for k in range(keys):
            assert c.lookup(k) == (m.key.index(k) if k in m.key else -1)


def test_errors(B):
    lib = B.load_library()
    import ctypes
    h = ctypes.c_void_p()
    assert lib.lora_slot_cache_create(0, ctypes.byref(h)) == -1
    assert lib.lora_slot_cache_create(B.MAX_SLOTS + 1, ctypes.byref(h)) == -1
    c = B.SlotCache(2)
    with pytest.raises(B.LoraError):
        c.acquire(-1)
    a, _, _ = c.acquire(10, pin=True)
    b, _, _ = c.acquire(11, pin=True)
    with pytest.raises(B.LoraError) as ei:   # both slots pinned: nothing changes
        c.acquire(12)
    assert ei.value.rc == -9
    assert c.lookup(10) == a and c.lookup(11) == b and c.lookup(12) == -1
    with pytest.raises(B.LoraError) as ei:
        c.unpin(2)
    assert ei.value.rc == -5
    c.unpin(a)
    with pytest.raises(B.LoraError):
        c.unpin(a)
    assert c.acquire(12) == (a, False, 10)   # the unpinned slot is the one reused
