"""End-to-end parity of moe_forward against the oracle on the GPU, through the C ABI.

Small shapes (several m-tiles, ragged token counts, ragged H/D, block sizes 16/48/128,
capacity, shared expert, router bias) compare every token; the five full-size workloads
compare a seeded sample of tokens (the oracle computes them one by one) plus the exact
align outputs and the logits of every token.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_block_b200 import configs, inputs as gen
from parity import check_forward, sample_tokens

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": configs.TINY,
    "prefill_small": configs.FLASHMOE_PREFILL.replace(name="prefill_small", T=515, H=512, D=384, E=16),
    "dsv3_small": configs.DSV3.replace(name="dsv3_small", T=300, H=1024, D=256, E=32, D_shared=256),
    "ragged_dims": configs.MoEWorkload("ragged_dims", T=77, H=320, D=200, E=5, top_k=2, block_m=48,
                                       D_shared=136, sigma_w=0.05),
    "skew_small": configs.SKEW.replace(name="skew_small", T=2000, H=512, D=256),
    "one_token": configs.DECODE.replace(name="one_token", T=1),
    "k_equals_E": configs.MoEWorkload("k_equals_E", T=200, H=256, D=128, E=4, top_k=4, block_m=16),
    # at most 16 tokens: the expert GEMMs take their small-tile shape
    "small_tokens_shared": configs.DSV3.replace(name="small_tokens_shared", T=12, H=512, D=256, E=16, top_k=4,
                                                D_shared=256),
    "small_tokens_ragged": configs.MoEWorkload("small_tokens_ragged", T=5, H=320, D=200, E=5, top_k=2,
                                               block_m=48, D_shared=136, sigma_w=0.05, capacity_factor=1.0),
}


def _layer(w, **kw):
    from mixture_experts_layer_block_b200.native import MoELayer
    return MoELayer.for_workload(w, **kw)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_forward_small_all_tokens(name):
    w = SMALL[name]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = _layer(w)
    res = check_forward(layer, w, inp)
    # a second call on the same handle reuses the workspace and must agree
    res2 = check_forward(layer, w, inp)
    assert res2["out_err"] <= 1e-2
    print(name, res)


@pytest.mark.parametrize("name", ["flashmoe_prefill", "dsv3", "decode", "skew", "skew_uniform"])
def test_forward_full_size_sampled(name):
    w = configs.WORKLOADS[name]
    torch.cuda.empty_cache()
    inp = gen.make_inputs(w, device="cuda")
    layer = _layer(w)
    tokens = sample_tokens(w.T, 48, seed=1)
    res = check_forward(layer, w, inp, tokens=tokens)
    print(name, res)
    del inp, layer
    torch.cuda.empty_cache()


def test_forward_smaller_T_than_max_tokens():
    w = SMALL["dsv3_small"]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = _layer(w, max_tokens=4 * w.T)
    check_forward(layer, w, inp)
    # a shorter batch on the same handle
    w2 = w.replace(T=33)
    inp2 = dict(inp, x=inp["x"][:33].contiguous())
    check_forward(layer, w2, inp2)


def test_forward_zero_tokens():
    w = SMALL["tiny"]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = _layer(w)
    out = torch.empty((0, w.H), dtype=torch.float32, device="cuda")
    layer.forward(inp["x"][:0], inp, out)
    torch.cuda.synchronize()
    assert layer.status() == (0, 0)


def test_forward_is_deterministic_in_routing():
    w = SMALL["skew_small"]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = _layer(w)
    outs, dbgs = [], []
    for _ in range(3):
        out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
        layer.forward(inp["x"], inp, out)
        dbgs.append(layer.debug_outputs(w.T, w.top_k, "cuda"))
        outs.append(out)
    torch.cuda.synchronize()
    for d in dbgs[1:]:
        for n in ("topk_ids", "sorted_ids", "expert_ids", "num_post_padded", "logits"):
            assert torch.equal(d[n], dbgs[0][n]), n
    # the combine sums in a run-dependent order: equal up to fp32 reassociation
    ref = outs[0].abs().max().item()
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 1e-5 * ref
