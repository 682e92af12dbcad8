"""Stage parity on the GPU through the C ABI: gating and align bit-exact against the oracle
on the same seeded inputs, router logits within the fp32 stage tolerance."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_block_b200 import inputs as gen
from oracle import oracle
from parity import STAGE_TOL, rel_err

pytestmark = pytest.mark.gpu


def _layer(E, k, block_m=16, max_tokens=1024, cf=0.0, H=256, D=128):
    from mixture_experts_layer_block_b200.native import MoELayer
    return MoELayer(H, D, E, k, block_m, max_tokens, capacity_factor=cf)


@pytest.mark.parametrize("E,k,ties", [(8, 2, False), (8, 8, True), (64, 2, False), (128, 8, True),
                                      (256, 8, False), (256, 8, True), (512, 4, True), (1024, 32, False),
                                      (33, 5, True)])
def test_gate_topk_bit_exact(E, k, ties):
    T = 777
    L = gen.make_logits(T, E, seed=E * 31 + k, ties=ties)
    layer = _layer(E, k, max_tokens=T)
    dev = torch.device("cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    layer.gate_topk(L.to(dev), k, ids, w)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.topk_softmax(L.double().numpy(), k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("dist", ["random", "alternating_empty", "skewed", "one_expert"])
@pytest.mark.parametrize("E,k,bm,T", [(8, 2, 16, 64), (64, 2, 128, 4096), (256, 8, 16, 16),
                                      (256, 8, 128, 4096), (128, 8, 48, 3001), (32, 4, 1, 517)])
@pytest.mark.parametrize("cf", [0.0, 1.0])
def test_align_bit_exact(dist, E, k, bm, T, cf):
    ids = gen.make_topk_ids(T, E, k, seed=T + E, dist=dist)
    layer = _layer(E, k, block_m=bm, max_tokens=T, cf=cf)
    dev = torch.device("cuda")
    sorted_ids = torch.full((layer.sorted_len(T, k),), -7, dtype=torch.int32, device=dev)
    expert_ids = torch.full((layer.blocks_len(T, k),), -7, dtype=torch.int32, device=dev)
    npp = torch.zeros((1,), dtype=torch.int32, device=dev)
    layer.align(ids.to(dev), sorted_ids, expert_ids, npp)
    torch.cuda.synchronize()
    ref = oracle.align(ids.numpy(), E, bm, oracle.capacity(T, k, E, cf))
    np.testing.assert_array_equal(sorted_ids.cpu().numpy(), ref["sorted_ids"])
    np.testing.assert_array_equal(expert_ids.cpu().numpy(), ref["expert_ids"])
    assert int(npp.item()) == ref["num_post_padded"]


def test_align_large_and_empty():
    dev = torch.device("cuda")
    for T, E, k, bm in [(16384, 128, 8, 128), (0, 64, 2, 16), (1, 256, 8, 16)]:
        ids = gen.make_topk_ids(T, E, k, seed=3, dist="skewed")
        layer = _layer(E, k, block_m=bm, max_tokens=max(T, 1))
        sorted_ids = torch.full((layer.sorted_len(T, k),), -7, dtype=torch.int32, device=dev)
        expert_ids = torch.full((layer.blocks_len(T, k),), -7, dtype=torch.int32, device=dev)
        npp = torch.full((1,), -7, dtype=torch.int32, device=dev)
        layer.align(ids.to(dev), sorted_ids, expert_ids, npp)
        torch.cuda.synchronize()
        ref = oracle.align(ids.numpy(), E, bm)
        np.testing.assert_array_equal(sorted_ids.cpu().numpy(), ref["sorted_ids"])
        np.testing.assert_array_equal(expert_ids.cpu().numpy(), ref["expert_ids"])
        assert int(npp.item()) == ref["num_post_padded"]


@pytest.mark.parametrize("T,H,E,bias", [(64, 256, 8, False), (300, 2048, 64, True),
                                        (1000, 7168, 256, False), (16, 2048, 256, True),
                                        (129, 4096, 128, True), (77, 320, 40, False)])
def test_router_logits_stage(T, H, E, bias):
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(T + H + E)
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    w = (0.02 * torch.randn((E, H), generator=g)).to(torch.bfloat16)
    b = torch.randn((E,), generator=g) if bias else None
    layer = _layer(E, min(E, 2), H=H, max_tokens=T)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    layer.router_logits(x.to(dev), w.to(dev), None if b is None else b.to(dev), logits)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x, w, None if b is None else b.numpy())
    assert rel_err(logits.cpu().numpy().astype(np.float64), ref) <= STAGE_TOL
