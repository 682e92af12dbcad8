"""MXFP8 experts on the GPU, through the C ABI, against the oracle's MXFP8 arithmetic.

The quantiser must match the oracle bit for bit (codes and scales, on bf16 inputs spanning the
exponent range, with zero blocks and saturating blocks); the MXFP8 forward must match the
oracle's MXFP8 layer within the output tolerance on small shapes (every token: several m-tiles,
ragged token counts, capacity drops, a shared expert, a router bias, H = 640 whose last 256-row
W_down box runs past the last expert) and on the full-size workloads (sampled tokens).

Both sides quantise x and the weights from the same bf16 values (identical decisions); h is
quantised from fp32 on both sides, from fp32 values that differ by the rounding of the two
accumulation orders, so an h code may differ where h sits on a rounding boundary; the output
tolerance (1e-2 of the largest output) covers such a code (one E4M3 step, at most 1/8 of one h
element, spread over a row of W_down) many times over.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_block_b200 import configs, inputs as gen
from oracle import oracle
from parity import check_forward

pytestmark = pytest.mark.gpu


def _native():
    from mixture_experts_layer_block_b200 import native
    return native


def sf_rows(sf: np.ndarray, R: int, K: int) -> np.ndarray:
    """Scale codes [R][K/32] from the atom layout of include/moe_b200.h."""
    r = np.arange(R)[:, None]
    b = np.arange(K // 32)[None, :]
    off = ((r // 128) * (K // 128) + b // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + b % 4
    return sf[off]


def _mixed_magnitudes(R, K, seed):
    g = torch.Generator().manual_seed(seed)
    mag = torch.exp2(torch.randint(-40, 40, (R, K // 32), generator=g).float()).repeat_interleave(32, dim=1)
    m = torch.randn(R, K, generator=g) * mag
    m[3, 64:96] = 0.0                       # an all-zero block
    m[5, :32] = 1e-38                       # a block of tiny normals
    m[7, 32:64] = torch.linspace(-1.0, 1.0, 32) * 3e38  # near the top of the range
    m[9, ::7] = 0.0
    return m.to(torch.bfloat16)


@pytest.mark.parametrize("R,K", [(128, 128), (256, 640), (384, 2048)])
def test_quantize_matches_oracle_bit_for_bit(R, K):
    native = _native()
    layer = native.MoELayer(256, 128, 8, 2, 16, 64)
    m = _mixed_magnitudes(R, K, seed=R + K)
    q, sf = layer.quantize_mxfp8(m.cuda())
    torch.cuda.synchronize()
    codes, scales = oracle.mx_quantize_bf16_rows(m)
    np.testing.assert_array_equal(q.cpu().numpy(), codes)
    np.testing.assert_array_equal(sf_rows(sf.cpu().numpy(), R, K), scales)
    layer.close()


def test_quantize_weight_tensor_views():
    """A 3-D expert tensor [E][D][H] is quantised as its [E*D][H] view."""
    native = _native()
    layer = native.MoELayer(256, 128, 8, 2, 16, 64)
    w = (0.02 * torch.randn(4, 128, 256, generator=torch.Generator().manual_seed(2))).to(torch.bfloat16)
    q, sf = layer.quantize_mxfp8(w.cuda())
    torch.cuda.synchronize()
    codes, scales = oracle.mx_quantize_bf16_rows(w.reshape(-1, 256))
    np.testing.assert_array_equal(q.cpu().numpy(), codes)
    np.testing.assert_array_equal(sf_rows(sf.cpu().numpy(), 512, 256), scales)
    layer.close()


MX_SMALL = {
    "tiny": configs.TINY,
    "prefill_small": configs.FLASHMOE_PREFILL.replace(name="prefill_small", T=515, H=512, D=384, E=16),
    "dsv3_small": configs.DSV3.replace(name="dsv3_small", T=300, H=1024, D=256, E=32, D_shared=256),
    "skew_small": configs.SKEW.replace(name="skew_small", T=2000, H=512, D=256),
    "one_token": configs.DECODE.replace(name="one_token", T=1),
    "decode": configs.DECODE,
    "h640": configs.MoEWorkload("h640", T=90, H=640, D=256, E=6, top_k=2, block_m=16, D_shared=128,
                                sigma_w=0.05),
}


def _setup(w, flags=0):
    native = _native()
    inp = gen.make_inputs(w, device="cuda")
    layer = native.MoELayer.for_workload(w, flags=native.MOE_FLAG_MXFP8 | flags)
    wq = layer.quantize_experts_mxfp8(inp)
    return layer, inp, wq


@pytest.mark.parametrize("name", sorted(MX_SMALL))
def test_forward_mxfp8_small_all_tokens(name):
    w = MX_SMALL[name]
    layer, inp, wq = _setup(w)
    res = check_forward(layer, w, inp, wq=wq)
    assert layer.query(8) == 4
    res2 = check_forward(layer, w, inp, wq=wq)
    assert res2["out_err"] <= 1e-2
    print(name, res)
    layer.close()


def test_forward_mxfp8_bf16_out():
    native = _native()
    w = MX_SMALL["dsv3_small"]
    layer, inp, wq = _setup(w, flags=native.MOE_FLAG_OUT_BF16)
    res = check_forward(layer, w, inp, wq=wq, out_dtype=torch.bfloat16)
    print(res)
    layer.close()


def test_forward_mxfp8_differs_from_bf16_by_quantisation_only():
    """The MXFP8 result is not the bf16 result (quantisation is applied), but it is close to it:
    the relative difference is of the order of E4M3's 2^-4 rounding, not larger."""
    w = MX_SMALL["prefill_small"]
    layer, inp, wq = _setup(w)
    out_mx = torch.empty(w.T, w.H, dtype=torch.float32, device="cuda")
    out_bf = torch.empty_like(out_mx)
    layer.forward_mxfp8(inp["x"], inp["W_router"], inp.get("bias"), wq, out_mx)
    layer.forward(inp["x"], inp, out_bf)
    torch.cuda.synchronize()
    d = (out_mx - out_bf).abs().max().item() / out_bf.abs().max().item()
    assert 1e-3 < d < 0.2, d
    layer.close()


@pytest.mark.parametrize("name", ["flashmoe_prefill", "dsv3", "skew"])
def test_forward_mxfp8_full_size_sampled(name):
    w = configs.WORKLOADS[name]
    layer, inp, wq = _setup(w)
    res = check_forward(layer, w, inp, tokens="tiles", min_tokens=128, wq=wq)
    assert res["compared_tokens"] >= 128 - res["near_ties"]
    print(name, res)
    layer.close()


def test_forward_mxfp8_zero_tokens_then_a_batch():
    """An empty batch launches nothing and leaves the handle usable."""
    w = MX_SMALL["tiny"]
    layer, inp, wq = _setup(w)
    out = torch.empty((0, w.H), dtype=torch.float32, device="cuda")
    layer.forward_mxfp8(inp["x"][:0], inp["W_router"], inp.get("bias"), wq, out)
    torch.cuda.synchronize()
    assert layer.status() == (0, 0)
    check_forward(layer, w, inp, wq=wq)
    layer.close()


def test_forward_mxfp8_is_deterministic():
    """Every slot's row is summed in slot order: repeated forwards agree bit for bit."""
    w = MX_SMALL["skew_small"]
    layer, inp, wq = _setup(w)
    outs = []
    for _ in range(3):
        out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
        layer.forward_mxfp8(inp["x"], inp["W_router"], inp.get("bias"), wq, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert layer.status() == (0, 0)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    layer.close()


@pytest.mark.parametrize("batch", [3, 64])
def test_forward_mxfp8_claim_batch(batch):
    """A claim batch changes which CTA runs a task, not its result: the oracle's result, and the
    same bits as one id per claim."""
    native = _native()
    w = MX_SMALL["dsv3_small"]
    outs = []
    for cb in (0, batch):
        inp = gen.make_inputs(w, device="cuda")
        layer = native.MoELayer.for_workload(w, flags=native.MOE_FLAG_MXFP8, claim_batch=cb)
        wq = layer.quantize_experts_mxfp8(inp)
        check_forward(layer, w, inp, wq=wq)
        out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
        layer.forward_mxfp8(inp["x"], inp["W_router"], inp.get("bias"), wq, out)
        torch.cuda.synchronize()
        assert layer.status() == (0, 0)
        outs.append(out)
        layer.close()
    assert torch.equal(outs[0], outs[1])


MX_FUSED = {
    "one_token": MX_SMALL["one_token"],
    "decode": MX_SMALL["decode"],                            # 256 experts top-8, router bias
    "small_tokens_shared": configs.DSV3.replace(name="small_tokens_shared", T=12, H=512, D=256, E=16, top_k=4,
                                                D_shared=256),  # the shared tile reads token-order xq
    "capacity_drops": configs.MoEWorkload("capacity_drops", T=9, H=384, D=256, E=6, top_k=2, block_m=16,
                                          sigma_w=0.05, capacity_factor=1.0),
    # the largest fused batch: 16 tokens x top-32 = 512 slots, every tile 16 rows, a shared expert
    "max_slots": configs.MoEWorkload("max_slots", T=16, H=256, D=128, E=32, top_k=32, block_m=16,
                                     D_shared=128, sigma_w=0.05),
    # the router bias moves the hit experts from seed to seed
    "decode_seed1": MX_SMALL["decode"].replace(name="decode_seed1", seed=1),
    "decode_seed2": MX_SMALL["decode"].replace(name="decode_seed2", seed=2),
}


@pytest.mark.parametrize("name", sorted(MX_FUSED))
def test_forward_mxfp8_small_batch_fused_and_unfused(name):
    """At most 16 tokens, MXFP8 experts: one fused launch by default (router slices, schedule,
    quantising gather, GEMMs, combine by the last down task of each column block) and the six
    kernels with MOE_FLAG_UNFUSED_SMALL; both match the oracle, and repeated fused forwards agree
    bit for bit."""
    native = _native()
    w = MX_FUSED[name]
    layer, inp, wq = _setup(w)
    assert layer.query(12) == 1
    res = check_forward(layer, w, inp, wq=wq)
    assert layer.query(11) == 1 and layer.query(8) == 4
    unfused, _, wq2 = _setup(w, flags=native.MOE_FLAG_UNFUSED_SMALL)
    check_forward(unfused, w, inp, wq=wq2)
    assert unfused.query(11) == 6 and unfused.query(12) == 0
    outs = []
    for _ in range(3):
        out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
        layer.forward_mxfp8(inp["x"], inp["W_router"], inp.get("bias"), wq, out)
        outs.append(out)
    torch.cuda.synchronize()
    assert layer.status() == (0, 0)
    assert all(torch.equal(o, outs[0]) for o in outs[1:])
    print(name, res)
    layer.close()
    unfused.close()
