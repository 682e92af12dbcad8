"""The allocation-free align entry point agrees with the handle-based one.

moe_align_block_size_noalloc serves callers that cannot let this library allocate device
memory (a runtime whose own allocator owns all of HBM, or a path that cannot afford a
cudaMalloc). It keeps its scratch in a fixed array inside the library, so two calls in a row
must each start from a clean state: this test runs two different inputs back to back through
the C ABI and compares every output with moe_align_block_size of a handle, exactly (they are
integer outputs). The file name makes pytest collect it last.
"""
import pytest
import torch

from mixture_experts_layer_block_b200 import inputs as gen

pytestmark = pytest.mark.gpu

CASES = [  # T, E, top_k, block_m, capacity_factor, distribution
    (4096, 64, 2, 128, 1.0, "random"),
    (16, 256, 8, 16, 0.0, "random"),
    (3001, 128, 8, 48, 0.0, "skewed"),
    (16384, 128, 8, 128, 0.0, "one_expert"),
]


def _run_handle(ids, E, k, bm, cf):
    from mixture_experts_layer_block_b200.native import MoELayer
    T = ids.shape[0]
    layer = MoELayer(256, 128, E, k, bm, max(T, 1), capacity_factor=cf)
    s = torch.full((layer.sorted_len(T, k),), -7, dtype=torch.int32, device="cuda")
    e = torch.full((layer.blocks_len(T, k),), -7, dtype=torch.int32, device="cuda")
    n = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    layer.align(ids, s, e, n)
    torch.cuda.synchronize()
    layer.close()
    return s, e, n


def _run_noalloc(ids, E, k, bm, cf):
    from mixture_experts_layer_block_b200.native import align_block_size_noalloc
    T = ids.shape[0]
    L = T * k + E * (bm - 1)
    s = torch.full((L,), -9, dtype=torch.int32, device="cuda")
    e = torch.full(((L + bm - 1) // bm,), -9, dtype=torch.int32, device="cuda")
    n = torch.full((1,), -9, dtype=torch.int32, device="cuda")
    align_block_size_noalloc(ids, E, bm, cf, s, e, n)
    return s, e, n


@pytest.mark.parametrize("first,second", [(0, 1), (2, 3), (3, 0)])
def test_noalloc_matches_handle_align_twice_in_a_row(first, second):
    runs = []
    for i in (first, second):
        T, E, k, bm, cf, dist = CASES[i]
        ids = gen.make_topk_ids(T, E, k, seed=11 + i, dist=dist).cuda()
        runs.append((ids, E, k, bm, cf, _run_noalloc(ids, E, k, bm, cf)))
    torch.cuda.synchronize()
    for ids, E, k, bm, cf, got in runs:
        ref = _run_handle(ids, E, k, bm, cf)
        for g, r, name in zip(got, ref, ("sorted_ids", "expert_ids", "num_post_padded")):
            assert torch.equal(g, r), name


def test_noalloc_empty_batch_between_two_batches():
    """T = 0 between two real batches: the empty call writes only sentinels (0), -1 block ids and
    P = 0, exactly like the handle align, and leaves nothing behind for the next call."""
    runs = []
    for i, T in ((1, None), (1, 0), (0, None)):
        T0, E, k, bm, cf, dist = CASES[i]
        T = T0 if T is None else T
        ids = gen.make_topk_ids(T, E, k, seed=21 + i, dist=dist).cuda()
        runs.append((ids, E, k, bm, cf, _run_noalloc(ids, E, k, bm, cf)))
    torch.cuda.synchronize()
    for ids, E, k, bm, cf, got in runs:
        ref = _run_handle(ids, E, k, bm, cf)
        for g, r, name in zip(got, ref, ("sorted_ids", "expert_ids", "num_post_padded")):
            assert torch.equal(g, r), name
    s0, e0, n0 = runs[1][5]
    assert int(n0.item()) == 0 and bool((s0 == 0).all()) and bool((e0 == -1).all())


def test_noalloc_rejects_sizes_beyond_its_limit():
    from mixture_experts_layer_block_b200.native import MOE_ERR_UNSUPPORTED, MoEError, align_block_size_noalloc
    ids = torch.zeros((8, 2), dtype=torch.int32, device="cuda")
    out = torch.zeros((4096,), dtype=torch.int32, device="cuda")
    with pytest.raises(MoEError) as e:
        align_block_size_noalloc(ids, 512, 16, 0.0, out, out, out[:1])  # 512 experts > 256
    assert e.value.code == MOE_ERR_UNSUPPORTED
