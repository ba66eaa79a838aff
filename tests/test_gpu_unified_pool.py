"""GPU: unified paging of KV-cache blocks and adapter weights in one pool.

Page "Multi-LoRA Serving in Production", section "Unified Paging
Architecture": all dynamic memory outside the base model is one pool of
fixed-size pages; KV-cache tensors and adapter weights are treated alike, and
adapter kernels gather weights from non-contiguous physical pages.  Here one
pool of 16-row pages (width d = d_in = d_out) first holds only KV blocks; a
random part of them is released, adapters are loaded into the scattered free
pages, the fused call runs against the fp64 oracle, and every KV page still
held must be untouched, bit for bit.  Evicting the adapters hands their pages
back to the KV side.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu


def test_kv_and_adapters_share_one_pool():
    import torch
    import heterogeneous_adapter_batching_b200 as H
    from tests import _util as U
    H.load_library()
    d = 1024
    wl = W.random_small(seed=77, T=90, d_in=d, d_out=d, S=10, ranks=(4, 16, 33, 64), p_none=0.1)
    need = int(sum(2 * ((a.rank + 15) // 16) for a in wl.adapters if a is not None))
    n_pages = need + 40
    layer = H.AdapterLayer(d, d, wl.S + 1, n_pages, n_pages, wl.T, shared_pool=True)   # one spare slot
    assert layer.pool_a is layer.pool_b
    # the whole pool as KV blocks, each filled with its own pattern
    kv = layer.alloc_pages(n_pages)
    assert H.lora_pool_free_pages(layer.pool_a) == 0
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    for p in kv.tolist():
        layer.page_rows(p).copy_(torch.randn((16, d), generator=g, device="cuda").to(torch.bfloat16))
    # release a scattered part of them; the adapters land in those pages
    rng = np.random.default_rng(8)
    freed = rng.choice(kv.numpy(), size=need, replace=False)
    layer.free_pages(torch.from_numpy(np.sort(freed).astype(np.int32)))
    kept = sorted(set(kv.tolist()) - set(freed.tolist()))
    kept_before = torch.stack([layer.page_rows(p).clone() for p in kept])
    for i, a in enumerate(wl.adapters):
        at = torch.from_numpy(W.bf16_bits(np.ascontiguousarray(a.A.T)).view(np.int16)).cuda()
        b = torch.from_numpy(W.bf16_bits(a.B).view(np.int16)).cuda()
        layer.load(i, a.rank, a.alpha, at, b)
    assert H.lora_pool_usage(layer.pool_a) == (need, n_pages - need)
    assert H.lora_pool_free_pages(layer.pool_a) == 0
    used = set(layer.page_table.cpu().numpy().ravel().tolist()) - {-1}
    assert used == set(freed.tolist())                      # only the released pages
    X, Y, ids = U.dev_inputs(wl)
    layer.apply(X, Y, ids)
    torch.cuda.synchronize()
    assert int(layer.err.item()) == 0
    ref, _ = U.oracle_full(wl)
    U.assert_parity(Y.cpu().numpy(), ref, wl.Y_base)
    kept_after = torch.stack([layer.page_rows(p) for p in kept])
    assert torch.equal(kept_before, kept_after)             # the KV blocks are untouched
    # a full pool refuses one more adapter (the spare slot), taking nothing
    with pytest.raises(H.LoraError):
        layer.load(wl.S, 16, 32.0, torch.zeros((16, d), dtype=torch.int16, device="cuda"),
                   torch.zeros((16, d), dtype=torch.int16, device="cuda"))
    assert H.lora_pool_usage(layer.pool_a) == (need, n_pages - need)
    # adapters out, KV in: the pages move back to the other tenant
    for i in range(wl.S):
        layer.evict(i)
    a_pages, o_pages = H.lora_pool_usage(layer.pool_a)
    assert a_pages == 0 and o_pages == n_pages - need
    more = layer.alloc_pages(need)
    assert H.lora_pool_usage(layer.pool_a) == (0, n_pages) and set(more.tolist()) == set(freed.tolist())
    torch.cuda.synchronize()
