"""GPU: the one-warp plan kernel for small batches writes the same plan as the
block-wide kernel, bit for bit: the whole workspace (header, slot offsets,
short-token list, gather jobs and their order), the caller's perm and
seg_start copies and the error bits, on batches with id = -1 tokens, ids out
of range, evicted slots, 1..128 slots and job sizes 1..16 (and a batch just
beyond the small kernel's slot limit)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import heterogeneous_adapter_batching_b200 as H
    H.load_library()
    return H


def _plan(H, ids_h, ranks_h, kernel):
    import torch
    T, S = len(ids_h), len(ranks_h)
    ids = torch.from_numpy(np.asarray(ids_h, np.int32)).cuda()
    ranks = torch.from_numpy(np.asarray(ranks_h, np.int32)).cuda()
    ws = torch.full((H.lora_workspace_size(T, S),), 0xA5, dtype=torch.uint8, device="cuda")
    perm = torch.full((max(T, 1),), -9, dtype=torch.int32, device="cuda")
    seg = torch.full((S + 1,), -9, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    H.lora_set_option(H.OPT_PLAN_KERNEL, kernel)
    try:
        H.lora_plan(ids, T, ranks, S, perm, seg, ws, err)
        torch.cuda.synchronize()
    finally:
        H.lora_set_option(H.OPT_PLAN_KERNEL, H.PLAN_AUTO)
    return ws.cpu().numpy(), perm.cpu().numpy(), seg.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("job_tokens", [1, 3, 16])
@pytest.mark.parametrize("seed,T,S", [(0, 1, 1), (1, 7, 3), (2, 31, 32), (3, 33, 5), (4, 64, 32), (5, 100, 128),
                                      (6, 127, 97), (7, 200, 128), (8, 256, 17), (9, 256, 64), (10, 64, 129)])
def test_small_plan_equals_general(H, seed, T, S, job_tokens):
    old = {k: H.lora_get_option(k) for k in (H.OPT_LONG_SEGMENT, H.OPT_DECODE_JOB_TOKENS)}
    H.lora_set_option(H.OPT_DECODE_JOB_TOKENS, job_tokens)
    H.lora_set_option(H.OPT_LONG_SEGMENT, 0)     # no long runs: the small kernel's domain
    try:
        rng = np.random.default_rng(seed)
        ranks = rng.choice(np.array([0, 4, 8, 16, 17, 33, 64]), size=S).astype(np.int32)
        # Zipf-like reuse of a few slots, id = -1 tokens, ids out of range
        ids = rng.choice(S, size=T, p=np.arange(1, S + 1)[::-1] / (S * (S + 1) / 2)).astype(np.int32)
        ids[rng.random(T) < 0.1] = -1
        if T > 4:
            ids[rng.integers(0, T)] = S + 2
        a = _plan(H, ids, ranks, H.PLAN_AUTO)
        b = _plan(H, ids, ranks, H.PLAN_GENERAL)
        assert a[3] == b[3]
        assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
        assert np.array_equal(a[0], b[0])
    finally:
        for k, v in old.items():
            H.lora_set_option(k, v)


def test_small_plan_apply_matches_oracle(H):
    """The fused call over a small-kernel plan (decode q_proj, 7B) against the oracle."""
    import workloads as W
    from tests import _util as U
    wl = W.decode_q_proj_7b(T=64)
    layer = U.make_layer(wl)
    X, Y, ids = U.dev_inputs(wl)
    layer.apply(X, Y, ids)
    import torch
    torch.cuda.synchronize()
    assert int(layer.err.item()) == 0
    ref, _ = U.oracle_full(wl)
    U.assert_parity(Y.cpu().numpy(), ref, wl.Y_base)
