"""End-to-end parity of moe_forward against the oracle on the GPU, through the C ABI.

Small shapes (several m-tiles, ragged token counts, ragged H/D, block sizes 16/48/128,
capacity, shared expert, router bias) compare every token; the five full-size workloads
compare every m-tile's first, last and a random row (the oracle computes them one by one) plus
the exact align outputs and the logits of every token; every comparison also checks the two
expert GEMMs and the combine stage by stage.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_block_b200 import configs, inputs as gen
from parity import check_forward

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
    # H = 640: a 512-column block of a row ends inside the first 256 columns of its second half
    "h640": configs.MoEWorkload("h640", T=90, H=640, D=192, E=6, top_k=2, block_m=16, D_shared=64,
                                sigma_w=0.05),
}


def _layer(w, **kw):
    from mixture_experts_layer_block_b200.native import MoELayer
    return MoELayer.for_workload(w, **kw)


def _flags():
    from mixture_experts_layer_block_b200 import native
    return {"pair": native.MOE_FLAG_PAIR_TILES, "single": native.MOE_FLAG_SINGLE_TILES,
            "general": native.MOE_FLAG_SINGLE_TILES | native.MOE_FLAG_NO_TAIL_TILES,
            "tail": native.MOE_FLAG_SINGLE_TILES | native.MOE_FLAG_TAIL_TILES,
            "two": native.MOE_FLAG_SINGLE_TILES | native.MOE_FLAG_TWO_TILES}


SHAPE_CODE = {"general": 0, "small": 1, "tail": 2, "pair": 3, "two": 5}


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


# Every shape of the expert GEMMs for batches of more than 16 tokens (256-row tiles on SM
# pairs; 128-row tiles on single SMs, with or without merged tails) on every small case: tiles
# of 1..256 rows, split between the two CTAs of a pair at every boundary the split rule has.
@pytest.mark.parametrize("shape", ["pair", "general", "tail", "two"])
@pytest.mark.parametrize("name", sorted(n for n, w in SMALL.items() if w.T > 16))
def test_forward_small_tile_shapes(name, shape):
    w = SMALL[name]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = _layer(w, flags=_flags()[shape])
    res = check_forward(layer, w, inp)
    assert layer.query(6) == (256 if shape == "pair" else 128)
    assert layer.query(8) == SHAPE_CODE[shape]
    res2 = check_forward(layer, w, inp)
    assert res2["out_err"] <= 1e-2
    print(name, shape, res)


@pytest.mark.parametrize("nrows", [17, 31, 32, 33, 64, 95, 127, 128, 129, 160, 200, 255, 256, 257, 300, 513])
def test_pair_tiles_one_expert(nrows):
    """Every token routed to expert 0 (top-1 of 2 experts with a large bias): one expert with
    nrows rows, i.e. pair tiles of every size around the 32-row box and 128-row half boundaries."""
    w = configs.MoEWorkload(f"one_expert_{nrows}", T=nrows, H=256, D=384, E=2, top_k=1, block_m=16,
                            D_shared=128, sigma_w=0.05)
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    inp["bias"] = torch.tensor([30.0, 0.0], dtype=torch.float32, device="cuda")
    layer = _layer(w, flags=_flags()["pair"])
    check_forward(layer, w, inp)
    assert layer.query(6) == 256


def test_tile_shape_selection():
    """Single SMs by default, SM pairs on request (when the device fits 2-CTA clusters), single
    SMs when both flags are given; two-tile task sets by default above 96 slots per expert unless
    the capacity holds an expert to one tile; the flags that ask for a shape win."""
    w2 = SMALL["skew_small"].replace(E=64, name="skew_small_64")  # 250 slots per expert
    inp2 = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w2).items()}
    f = _flags()
    layer = _layer(w2)
    check_forward(layer, w2, inp2)
    assert layer.query(6) == 128 and layer.query(1) == layer.query(0)
    assert layer.query(8) == SHAPE_CODE["two"]  # more than 96 slots per expert: two-tile tasks
    wide = w2.replace(E=16, name="skew_small_16")  # 1000 slots per expert
    inp3 = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(wide).items()}
    layer = _layer(wide)
    check_forward(layer, wide, inp3)
    assert layer.query(8) == SHAPE_CODE["two"]
    # a capacity of at most one tile per expert, or a light load: the general shape
    capped = w2.replace(capacity_factor=0.5, name="skew_small_capped")  # 125 slots per expert
    layer = _layer(capped)
    check_forward(layer, capped, inp2)
    assert layer.query(8) == SHAPE_CODE["general"]
    light = w2.replace(E=256, name="skew_small_256")  # 62.5 slots per expert
    inp4 = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(light).items()}
    layer = _layer(light)
    check_forward(layer, light, inp4)
    assert layer.query(8) == SHAPE_CODE["general"]
    layer = _layer(w2, flags=f["tail"])
    check_forward(layer, w2, inp2)
    assert layer.query(8) == SHAPE_CODE["tail"]
    layer = _layer(w2, flags=f["general"])
    check_forward(layer, w2, inp2)
    assert layer.query(8) == SHAPE_CODE["general"]
    layer = _layer(w2, flags=f["pair"])
    check_forward(layer, w2, inp2)
    assert layer.query(7) > 0 and layer.query(6) == 256 and layer.query(1) == layer.query(7)
    layer = _layer(w2, flags=f["pair"] | f["single"])
    check_forward(layer, w2, inp2)
    assert layer.query(6) == 128


FULL_SIZE = {n: configs.WORKLOADS[n] for n in ("flashmoe_prefill", "dsv3", "decode", "skew", "skew_uniform")}
# the decode layer's per-expert router bias moves the hit experts from seed to seed
FULL_SIZE["decode_seed1"] = configs.DECODE.replace(seed=1)
FULL_SIZE["decode_seed2"] = configs.DECODE.replace(seed=2)


@pytest.mark.parametrize("name", sorted(FULL_SIZE))
def test_forward_full_size_tiles(name):
    """The full-size workloads in the launch configuration the benchmark times: routing and
    align exact for every token; element-wise outputs for every m-tile's first, last and a
    random row (and every shared-expert tile's), at least 512 tokens; and the stage-by-stage
    checks of GEMM1 + SwiGLU, GEMM2 and the combine on the same tiles' rows."""
    w = FULL_SIZE[name]
    torch.cuda.empty_cache()
    inp = gen.make_inputs(w, device="cuda")
    layer = _layer(w)
    res = check_forward(layer, w, inp, tokens="tiles", min_tokens=512)
    assert res["compared_tokens"] >= min(512, w.T) - res["near_ties"]
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
    # each token's rows are summed in slot order whatever the task schedule: bit for bit equal
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("name", ["tiny", "dsv3_small", "ragged_dims", "one_token", "small_tokens_shared"])
def test_forward_bf16_out(name):
    """MOE_FLAG_OUT_BF16: the combine's fp32 sums rounded once to bf16. Bit-identical to the fp32
    output rounded to nearest even (same routing, same per-slot rows, same summation order), and
    within tolerance of the oracle; the host-staged path returns the same bytes."""
    from mixture_experts_layer_block_b200 import native
    w = SMALL[name]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    l16 = _layer(w, flags=native.MOE_FLAG_OUT_BF16 | native.MOE_FLAG_HOST_STAGING)
    check_forward(l16, w, inp, out_dtype=torch.bfloat16)
    l32 = _layer(w)
    o32 = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
    o16 = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    l32.forward(inp["x"], inp, o32)
    l16.forward(inp["x"], inp, o16)
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16))
    oh = torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory()
    l16.forward_host(inp["x"].cpu().pin_memory(), inp, oh)
    assert torch.equal(oh, o16.cpu())
    with pytest.raises(TypeError):
        l16.forward(inp["x"], inp, o32)


@pytest.mark.parametrize("shape", ["tail", "general", "two"])
@pytest.mark.parametrize("nrows", [129, 140, 160, 161, 200, 225, 256, 288, 289, 300, 416, 417, 513])
def test_single_sm_merged_tails_one_expert(nrows, shape):
    """Every token routed to expert 0 (top-1 of 2 with a large bias) and the shared expert over
    the same tokens: runs of 128-row tiles ending in tails of 1..128 rows. Tail shape: a tail of at
    most 32 rows rides in the tasks of the tile before it (an odd run starts with a single tile so
    the tail closes a pair), a longer one keeps its own tasks. Two-tile shape: every pair of tiles
    (second tile of any size, loaded as 32-row boxes up to 96 rows) runs as one task set."""
    w = configs.MoEWorkload(f"tails_{nrows}", T=nrows, H=256, D=384, E=2, top_k=1, block_m=16,
                            D_shared=128, sigma_w=0.05)
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    inp["bias"] = torch.tensor([30.0, 0.0], dtype=torch.float32, device="cuda")
    layer = _layer(w, flags=_flags()[shape])
    check_forward(layer, w, inp)
    assert layer.query(8) == SHAPE_CODE[shape]
    check_forward(layer, w, inp)  # the same handle again


# claim batches: a CTA takes this many consecutive task ids per atomic on the counter
@pytest.mark.parametrize("batch", [2, 5, 64])
@pytest.mark.parametrize("name,shape", [("dsv3_small", "general"), ("dsv3_small", "two"), ("skew_small", "tail"),
                                        ("prefill_small", "pair"), ("small_tokens_shared", None),
                                        ("small_tokens_ragged", "unfused")])
def test_forward_claim_batch(name, shape, batch):
    """Every claim batch gives the oracle's result, and the same bits as one id per claim: the
    batch changes which CTA runs a task, never what the task computes or the combine order."""
    from mixture_experts_layer_block_b200 import native
    w = SMALL[name]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    flags = native.MOE_FLAG_UNFUSED_SMALL if shape == "unfused" else _flags().get(shape, 0)
    outs = []
    for cb in (0, batch):
        layer = _layer(w, flags=flags, claim_batch=cb)
        check_forward(layer, w, inp)
        o = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
        layer.forward(inp["x"], inp, o)
        torch.cuda.synchronize()
        assert layer.status() == (0, 0)
        outs.append(o)
    assert torch.equal(outs[0], outs[1])


STATIC_CASES = {
    "tiny": SMALL["tiny"],                      # 8 experts: 18 CTAs each
    "dsv3_small": SMALL["dsv3_small"],          # 32 experts + shared: 4 CTAs each
    "skew_small": SMALL["skew_small"],          # 128 experts: one CTA each, 20 idle
    "small_tokens_shared": SMALL["small_tokens_shared"],  # small-tile shape
    "many_experts": configs.MoEWorkload("many_experts", T=200, H=256, D=128, E=300, top_k=4,
                                        block_m=16, D_shared=128, sigma_w=0.05),  # 301 > 148 CTAs
}


@pytest.mark.parametrize("name", sorted(STATIC_CASES))
def test_forward_static_quota(name):
    """MOE_FLAG_STATIC_QUOTA (the static per-expert SM quota baseline): same results as the
    dynamic queue, for fewer experts than CTAs, one CTA per expert and more experts than CTAs."""
    from mixture_experts_layer_block_b200 import native
    w = STATIC_CASES[name]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    for extra in (0, native.MOE_FLAG_TAIL_TILES):
        layer = _layer(w, flags=native.MOE_FLAG_STATIC_QUOTA | extra)
        check_forward(layer, w, inp)
        check_forward(layer, w, inp)


def test_forward_host_async_pipelined():
    """moe_forward_host_async: back-to-back calls on different batches (copies overlapping the
    neighbouring forwards) give exactly the synchronous call's outputs; a synchronous call after
    queued ones waits for them first."""
    from mixture_experts_layer_block_b200 import native
    w = SMALL["dsv3_small"]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = _layer(w, flags=native.MOE_FLAG_HOST_STAGING)
    xs = [gen.make_x(w.replace(seed=w.seed + i)).pin_memory() for i in range(5)]
    ref = []
    for x in xs:
        o = torch.empty((w.T, w.H), dtype=torch.float32).pin_memory()
        layer.forward_host(x, inp, o)
        ref.append(o.clone())
    outs = [torch.full((w.T, w.H), float("nan"), dtype=torch.float32).pin_memory() for _ in xs]
    stream = torch.cuda.current_stream()
    for x, o in zip(xs, outs):
        layer.forward_host_async(x, inp, o, stream=stream)
    layer.forward_host_join(stream=stream, block=True)
    for o, r in zip(outs, ref):
        assert torch.equal(o, r)
    # queued calls, then a synchronous one: every result lands
    layer.forward_host_async(xs[0], inp, outs[0], stream=stream)
    last = torch.empty((w.T, w.H), dtype=torch.float32).pin_memory()
    layer.forward_host(xs[1], inp, last)
    layer.forward_host_join(block=True)
    assert torch.equal(outs[0], ref[0]) and torch.equal(last, ref[1])
    rc, st = layer.status()
    assert rc == 0 and st == 0


FUSED_CASES = {
    "one_token": SMALL["one_token"],
    "small_tokens_shared": SMALL["small_tokens_shared"],
    "small_tokens_ragged": SMALL["small_tokens_ragged"],   # capacity drops, ragged H and D
    "decode": configs.DECODE,                               # 256 experts top-8, router bias
    "sixteen_rows_one_expert": configs.MoEWorkload("sixteen_rows_one_expert", T=16, H=256, D=384, E=2, top_k=1,
                                                   block_m=16, D_shared=128, sigma_w=0.05),
    "many_experts_few_ctas": configs.MoEWorkload("many_experts_few_ctas", T=9, H=512, D=256, E=200, top_k=6,
                                                 block_m=16, sigma_w=0.05),
    # the largest fused batch: 16 tokens x top-32 = 512 slots, every tile 16 rows, a shared expert
    "max_slots": configs.MoEWorkload("max_slots", T=16, H=256, D=128, E=32, top_k=32, block_m=16,
                                     D_shared=128, sigma_w=0.05),
}


@pytest.mark.parametrize("name", sorted(FUSED_CASES))
def test_small_batch_fused_and_unfused(name):
    """Batches of at most 16 tokens run as one fused launch by default (router slices, gating and
    align in the last CTA, gather, expert GEMMs, combine by the last down task of each column
    block) and as the six kernels with MOE_FLAG_UNFUSED_SMALL: both match the oracle stage by
    stage, and repeated fused forwards agree bit for bit."""
    from mixture_experts_layer_block_b200 import native
    w = FUSED_CASES[name]
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    if name == "sixteen_rows_one_expert":
        inp["bias"] = torch.tensor([30.0, 0.0], dtype=torch.float32, device="cuda")
    fused = _layer(w)
    assert fused.query(12) == 1
    res = check_forward(fused, w, inp)
    assert fused.query(11) == 1 and fused.query(8) == SHAPE_CODE["small"]
    unfused = _layer(w, flags=native.MOE_FLAG_UNFUSED_SMALL)
    check_forward(unfused, w, inp)
    assert unfused.query(11) == 6 and unfused.query(12) == 0
    outs = []
    for _ in range(3):
        o = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
        fused.forward(inp["x"], inp, o)
        outs.append(o)
    torch.cuda.synchronize()
    assert fused.status() == (0, 0)
    assert all(torch.equal(o, outs[0]) for o in outs[1:])
    print(name, res)


def test_small_batch_fused_stage_times_and_smaller_batches():
    """The fused launch on a handle sized for more tokens, with shrinking batches in a row (the
    per-forward counters start afresh each time), and its stage timing (all in the GEMM slot)."""
    from mixture_experts_layer_block_b200 import native
    w = configs.DECODE
    inp = gen.make_inputs(w, device="cuda")
    layer = _layer(w, flags=native.MOE_FLAG_STAGE_TIMING, max_tokens=64)
    for T in (16, 7, 1, 16):
        wt = w.replace(T=T)
        check_forward(layer, wt, dict(inp, x=inp["x"][:T].contiguous()))
        assert layer.query(11) == 1
    ms = layer.stage_times()
    assert ms[4] > 0 and all(abs(v) < 0.01 for i, v in enumerate(ms) if i != 4)
