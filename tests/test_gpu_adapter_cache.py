"""GPU: AdapterCache keeps a working set of adapters resident through the LRU
slot manager; batches whose adapters are evicted and reloaded still match the
fp64 oracle (page "LoRA Adapters at Serve Time with vLLM Multi-LoRA", section
"The Inference Mechanism: A Worked Scenario", step "Eviction")."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu


def test_working_set_through_the_slot_manager():
    import torch
    import heterogeneous_adapter_batching_b200 as H
    from oracle import build_oracle as OC
    H.load_library()
    d_in, d_out, S, n_adapters = 256, 320, 4, 10
    rng = np.random.default_rng([91, 1])
    ranks = rng.choice(np.array([1, 4, 16, 33, 64]), size=n_adapters)
    ad = W.Adapters(91, d_in, d_out, ranks, cache=True)
    host = {}
    for k in range(n_adapters):
        a = ad[k]
        at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16))
        b = torch.from_numpy(W.bf16_bits(a.B).view(np.int16))
        host[k] = (at, b, a.alpha)
    pages = S * 4 + 4
    layer = H.AdapterLayer(d_in, d_out, S, pages, pages, 64)
    cache = H.AdapterCache(layer, host)
    batches = [[0, 1, 2, 0, -1, 3], [4, 4, 2, 3], [6, 7, 8, 9, 9], [0, 1, 2, 3, 0]]
    for bi, keys in enumerate(batches):
        T = len(keys)
        X = W.bf16_round(rng.standard_normal((T, d_in), dtype=np.float32) / np.float32(np.sqrt(d_in)))
        Yb = rng.standard_normal((T, d_out), dtype=np.float32)
        ids, pinned = cache.map_batch(keys)
        Xd = torch.from_numpy(W.bf16_bits(X).view(np.int16)).cuda().view(torch.bfloat16)
        Yd = torch.from_numpy(Yb.copy()).cuda()
        layer.err.zero_()
        layer.apply(Xd, Yd, ids)
        torch.cuda.synchronize()
        cache.release(pinned)
        assert int(layer.err.item()) == 0
        # the reference uses the adapters by key
        A = [ad[k].A for k in range(n_adapters)]
        Bm = [ad[k].B for k in range(n_adapters)]
        sc = ad.alpha_of / ranks.astype(np.float32)      # each adapter's own alpha / r
        ref, _ = OC.lora_apply_c(X, Yb, np.array(keys, dtype=np.int32), A, Bm, sc)
        got = Yd.cpu().numpy()
        assert np.all(np.abs(got - ref) <= 2e-3 + 1e-2 * np.abs(ref)), bi
        for k in set(keys) - {-1}:
            assert cache.slots.lookup(k) >= 0
    # batch 2: 4 replaces the least recent (0), 2 and 3 hit; batch 3 pushes out
    # 1, 4, 2, 3; batch 4 reloads 0..3
    assert cache.slots.stats() == (2, 13, 9)
