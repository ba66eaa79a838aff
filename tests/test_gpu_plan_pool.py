"""GPU: the segment plan and the page pool, checked bit-exactly."""
import numpy as np
import pytest

import workloads as W
from oracle import lora_oracle as O
from tests import _util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    return H


def _plan(H, ids_h, ranks_h):
    import torch
    S = len(ranks_h)
    T = len(ids_h)
    ids = torch.from_numpy(np.asarray(ids_h, np.int32)).cuda()
    ranks = torch.from_numpy(np.asarray(ranks_h, np.int32)).cuda()
    ws = torch.empty(H.lora_workspace_size(T, S), dtype=torch.uint8, device="cuda")
    perm = torch.full((max(T, 1),), -9, dtype=torch.int32, device="cuda")
    seg = torch.full((S + 1,), -9, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    H.lora_plan(ids, T, ranks, S, perm, seg, ws, err)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), seg.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("seed,T,S", [(0, 1, 1), (1, 64, 32), (2, 1000, 7), (3, 17000, 6), (4, 5000, 4096),
                                      (5, 1024, 512), (6, 33, 1000), (7, 40000, 300)])
def test_plan_bit_exact(H, seed, T, S):
    rng = np.random.default_rng(seed)
    ranks = rng.choice(np.array([0, 4, 16, 64]), size=S, p=[0.1, 0.3, 0.3, 0.3]).astype(np.int32)
    ids = rng.integers(-1, S, size=T).astype(np.int32)
    if T > 10:
        ids[rng.integers(0, T, size=3)] = [S, -3, S + 100]
    perm, seg, err = _plan(H, ids, ranks)
    rperm, rseg, rerr = O.segment_plan(ids, ranks)
    n = len(rperm)
    assert np.array_equal(perm[:n], rperm)
    assert np.array_equal(seg, rseg)
    assert err == rerr


def test_plan_all_invalid_and_zipf(H):
    perm, seg, err = _plan(H, np.full(100, -1, np.int32), np.full(8, 16, np.int32))
    assert np.array_equal(seg, np.zeros(9)) and err == 0
    wl = W.mixed_mlp(which="up")
    perm, seg, err = _plan(H, wl.ids, wl.ranks())
    rperm, rseg, _ = O.segment_plan(wl.ids, wl.ranks())
    assert np.array_equal(perm, rperm) and np.array_equal(seg, rseg)


def test_pool_round_trip_shuffled_pages(H):
    import torch
    wl = W.random_small(seed=21, T=4, d_in=200, d_out=328, S=9, ranks=(1, 4, 15, 16, 17, 40, 64))
    layer = U.make_layer(wl)
    pt = layer.page_table.cpu().numpy()
    assert np.array_equal(pt, wl.page_ids)
    assert np.array_equal(layer.ranks.cpu().numpy(), wl.ranks())
    assert np.array_equal(layer.scales.cpu().numpy(), wl.scales_f32())
    for i in range(wl.S):
        a = wl.adapters[i]
        for m, (mat, width, pool) in enumerate(((a.A.T, wl.d_in, layer.pool_a), (a.B, wl.d_out, layer.pool_b))):
            out = torch.empty(width, dtype=torch.int16, device="cuda")
            for k in range(a.rank):
                H.lora_pool_read_row(pool, layer.page_table, wl.S, i, m, k, out)
                got = out.cpu().numpy().view(np.uint16)
                assert np.array_equal(got, W.bf16_bits(np.ascontiguousarray(mat[k])))
    # raw pool bytes: physical row = page * 16 + k % 16 (llms.blog, "Unified Paging Architecture")
    raw_b = layer.buf_b.view(torch.int16).cpu().numpy().view(np.uint16)
    for i in range(wl.S):
        a = wl.adapters[i]
        for k in range(a.rank):
            row = O.page_row(wl.page_ids[i, 1], k)
            assert np.array_equal(raw_b[row], W.bf16_bits(a.B[k]))
        # the unused rows of the last page are zero
        last = (a.rank - 1) // 16
        for k in range(a.rank, (last + 1) * 16):
            assert not raw_b[int(wl.page_ids[i, 1, last]) * 16 + k % 16].any()


def test_pool_free_list_oom_and_reuse(H):
    import torch
    d = 64
    buf = torch.empty((5 * 16, d), dtype=torch.bfloat16, device="cuda")
    pool = H.lora_pool_create(buf, d)
    assert H.lora_pool_num_pages(pool) == 5 and H.lora_pool_free_pages(pool) == 5
    S = 4
    pt = torch.full((S, 2, 4), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros(S, dtype=torch.float32, device="cuda")
    rk = torch.zeros(S, dtype=torch.int32, device="cuda")
    a = torch.zeros((40, d), dtype=torch.int16, device="cuda")
    with pytest.raises(H.LoraError, match="POOL_OOM"):
        H.lora_pool_load(pool, pool, 0, S, 40, 80.0, a, a, None, pt, sc, rk)     # 3 + 3 pages > 5
    assert H.lora_pool_free_pages(pool) == 5      # nothing leaked
    H.lora_pool_load(pool, pool, 1, S, 16, 32.0, a[:16], a[:16], None, pt, sc, rk)
    assert H.lora_pool_free_pages(pool) == 3
    H.lora_pool_evict(pool, pool, 1, S, pt, sc, rk)
    assert H.lora_pool_free_pages(pool) == 5


def test_pool_errors(H):
    import torch
    d = 64
    buf = torch.empty((7 * 16, d), dtype=torch.bfloat16, device="cuda")
    pool = H.lora_pool_create(buf, d)
    S = 4
    pt = torch.full((S, 2, 4), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros(S, dtype=torch.float32, device="cuda")
    rk = torch.zeros(S, dtype=torch.int32, device="cuda")
    a = torch.zeros((40, d), dtype=torch.int16, device="cuda")
    with pytest.raises(H.LoraError, match="POOL_OOM"):
        H.lora_pool_load(pool, pool, 0, S, 64, 1.0, a.new_zeros((64, d)), a.new_zeros((64, d)), None, pt, sc, rk)
    assert H.lora_pool_free_pages(pool) == 7
    H.lora_pool_load(pool, pool, 0, S, 40, 80.0, a, a, None, pt, sc, rk)
    assert H.lora_pool_free_pages(pool) == 1
    with pytest.raises(H.LoraError, match="BAD_SLOT"):   # occupied slot
        H.lora_pool_load(pool, pool, 0, S, 4, 8.0, a[:4], a[:4], None, pt, sc, rk)
    with pytest.raises(H.LoraError, match="BAD_RANK"):
        H.lora_pool_load(pool, pool, 1, S, 65, 8.0, a, a, None, pt, sc, rk)
    with pytest.raises(H.LoraError, match="BAD_SLOT"):
        H.lora_pool_load(pool, pool, S, S, 4, 8.0, a[:4], a[:4], None, pt, sc, rk)
    H.lora_pool_evict(pool, pool, 0, S, pt, sc, rk)
    assert H.lora_pool_free_pages(pool) == 7
    assert int(rk[0].item()) == 0 and (pt[0].cpu().numpy() == -1).all()
    with pytest.raises(H.LoraError, match="BAD_SLOT"):   # nothing to evict
        H.lora_pool_evict(pool, pool, 0, S, pt, sc, rk)
    other = torch.empty((2 * 16, 128), dtype=torch.bfloat16, device="cuda")
    pool_w = H.lora_pool_create(other, 128)
    ws = torch.empty(H.lora_workspace_size(4, S), dtype=torch.uint8, device="cuda")
    X = torch.zeros((4, d), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    ids = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(H.LoraError, match="WIDTH_MISMATCH"):
        H.lora_apply(X, Y, 4, d, 64, ids, S, rk, sc, pt, pool_w, pool, ws)
    with pytest.raises(H.LoraError, match="WORKSPACE"):
        H.lora_apply(X, Y, 4, d, 64, ids, S, rk, sc, pt, pool, pool, ws[:16])
