"""GPU: asynchronous prefetch of adapters into the paged pool on a copy stream.

Page "Multi-LoRA Serving in Production", section "Production Engineering
Guidelines", "Asynchronous Prefetching and Request Queuing": a cache miss
starts a non-blocking H2D copy from pinned host memory and the request waits
until it lands, while the running batches continue.  Each batch's adapters are
prefetched while the previous batch computes (the host never synchronises
between them); every batch is checked against the fp64 oracle, through
evictions and reloads.  A second test measures how much of the loads' time
hides under compute.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu


def _host_adapters(seed, d_in, d_out, ranks):
    import torch
    ad = W.Adapters(seed, d_in, d_out, ranks, cache=True)
    host = {}
    for k in range(len(ranks)):
        a = ad[k]
        at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16)).pin_memory()
        b = torch.from_numpy(W.bf16_bits(a.B).view(np.int16)).pin_memory()
        host[k] = (at, b, a.alpha)
    return ad, host


def test_prefetch_overlapped_batches_match_oracle():
    import torch
    import heterogeneous_adapter_batching_b200 as H
    from oracle import build_oracle as OC
    H.load_library()
    d_in, d_out, S, n_ad = 1024, 2048, 6, 14
    rng = np.random.default_rng([92, 1])
    ranks = rng.choice(np.array([4, 16, 33, 64]), size=n_ad)
    ad, host = _host_adapters(92, d_in, d_out, ranks)
    layer = H.AdapterLayer(d_in, d_out, S, S * 4 + 4, S * 4 + 4, 64)
    pf = H.AdapterPrefetcher(layer, host)
    compute = torch.cuda.Stream()
    # at most 3 distinct adapters per batch: two pinned batches fit in 6 slots
    batches = []
    for i in range(10):
        keys = rng.choice(n_ad, size=3, replace=False)
        toks = rng.choice(np.concatenate([keys, [-1]]), size=40)
        batches.append(toks.astype(np.int64))
    Xs = [W.bf16_round(rng.standard_normal((40, d_in), dtype=np.float32) / np.float32(np.sqrt(d_in)))
          for _ in batches]
    Ybs = [rng.standard_normal((40, d_out), dtype=np.float32) for _ in batches]
    Xd = [torch.from_numpy(W.bf16_bits(x).view(np.int16)).cuda().view(torch.bfloat16) for x in Xs]
    Yd = [torch.from_numpy(y.copy()).cuda() for y in Ybs]
    torch.cuda.synchronize()
    tickets = [pf.prefetch(batches[0])]
    misses = tickets[0].misses
    for i in range(len(batches)):
        if i + 1 < len(batches):
            tickets.append(pf.prefetch(batches[i + 1]))        # next batch's loads overlap this batch
            misses += tickets[-1].misses
        ids = pf.begin(tickets[i], compute)
        layer.apply(Xd[i], Yd[i], ids, stream=compute)
        pf.end(tickets[i], compute)
    torch.cuda.synchronize()
    assert int(layer.err.item()) == 0
    assert misses > S and pf.slots.stats()[2] > 0              # evictions and reloads happened
    A = [ad[k].A for k in range(n_ad)]
    Bm = [ad[k].B for k in range(n_ad)]
    sc = ad.alpha_of / ranks.astype(np.float32)
    for i, keys in enumerate(batches):
        ref, _ = OC.lora_apply_c(Xs[i], Ybs[i], keys.astype(np.int32), A, Bm, sc)
        got = Yd[i].cpu().numpy()
        assert np.all(np.abs(got - ref) <= 2e-3 + 1e-2 * np.abs(ref)), i


def test_prefetch_loads_hide_under_compute():
    """Loads of 24 rank-64 adapters (8B MLP widths) on the copy stream while the
    compute stream runs a batch of 128 distinct adapters: the pair takes less
    time than the two one after the other."""
    import torch
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    d_in, d_out = 4096, 14336
    wl = W.sweep_8b(T=256, regime="distinct", pool=128)
    from tests import _util as U
    work = U.make_layer(wl)
    X, Y, ids = U.dev_inputs(wl)
    n_ad = 24
    _, host = _host_adapters(93, d_in, d_out, np.full(n_ad, 64))
    target = H.AdapterLayer(d_in, d_out, n_ad, n_ad * 4, n_ad * 4, 16)
    pf = H.AdapterPrefetcher(target, host)
    compute = torch.cuda.Stream()

    def run_compute(reps=12):
        with torch.cuda.stream(compute):
            for _ in range(reps):
                work.apply(X, Y, ids, stream=compute)

    def timed(fn):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(compute)
        pf.copy.wait_event(e0)
        fn()
        compute.wait_stream(pf.copy)
        e1.record(compute)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def load_all():
        t = pf.prefetch(list(range(n_ad)))
        pf.end(t, pf.copy)
        for k in range(n_ad):                                   # make the next round miss again
            s = pf.slots.lookup(k)
            target.evict(s, stream=pf.copy)
            pf.slots.invalidate(s)

    run_compute(2)
    load_all()
    t_c = timed(run_compute)
    t_l = timed(load_all)
    t_both = timed(lambda: (load_all(), run_compute()))
    hidden = (t_c + t_l - t_both) / min(t_c, t_l)
    assert hidden > 0.3, (t_c, t_l, t_both)
