"""The parity machinery itself, on the CPU: the certification of routing near-ties, the token
sampler, and the seeded input generator that both the oracle and the CUDA path read."""
import numpy as np
import torch

from mixture_experts_layer_block_b200 import configs, inputs as gen
from parity import certified_routing, sample_tokens


def _logits():
    # token 0: clear order 3 > 1 > 0 > 2; token 1: experts 0 and 2 within 1e-9 of each other
    return np.array([[0.5, 2.0, -1.0, 3.0], [1.0, -2.0, 1.0 - 1e-9, 0.0]])


def test_identical_routing_is_status_0():
    L = _logits()
    absdot = np.ones_like(L)
    ids = np.array([[3, 1], [0, 2]], dtype=np.int32)
    status, ref = certified_routing(ids, L, absdot, H=64)
    assert status.tolist() == [0, 0]
    np.testing.assert_array_equal(ref, ids)


def test_swap_inside_the_error_bound_is_certified():
    L = _logits()
    absdot = np.ones_like(L)  # bound 4 * 64 * 2^-24 ~ 1.5e-5, far above the 1e-9 gap
    ids = np.array([[3, 1], [2, 0]], dtype=np.int32)
    status, _ = certified_routing(ids, L, absdot, H=64)
    assert status.tolist() == [0, 1]


def test_difference_outside_the_bound_is_rejected():
    L = _logits()
    absdot = np.ones_like(L)
    for bad in ([[1, 3], [0, 2]], [[3, 0], [0, 2]], [[3, 3], [0, 2]], [[3, 7], [0, 2]]):
        status, _ = certified_routing(np.array(bad, dtype=np.int32), L, absdot, H=64)
        assert status[0] == 2, bad


def test_tiny_bound_rejects_even_near_ties():
    L = _logits()
    absdot = np.full_like(L, 1e-12)
    status, _ = certified_routing(np.array([[3, 1], [2, 0]], dtype=np.int32), L, absdot, H=64)
    assert status[1] == 2


def test_sample_tokens_covers_both_ends():
    s = sample_tokens(4096, 64, seed=3)
    assert np.all(np.diff(s) > 0) and s[0] == 0 and s[-1] == 4095
    assert 48 <= s.size <= 64
    assert sample_tokens(10, 64).tolist() == list(range(10))


def test_inputs_are_seeded_and_deterministic():
    w = configs.TINY
    a, b = gen.make_inputs(w), gen.make_inputs(w)
    for k in a:
        if a[k] is None:
            assert b[k] is None
            continue
        assert torch.equal(a[k], b[k]), k
    c = gen.make_inputs(w.replace(seed=1))
    assert not torch.equal(a["x"], c["x"]) and not torch.equal(a["W_up"], c["W_up"])
    assert a["x"].dtype == torch.bfloat16 and a["W_up"].shape == (w.E, w.D, w.H)
    assert a["W_down"].shape == (w.E, w.H, w.D)


def test_inputs_have_the_stated_scale():
    w = configs.FLASHMOE_PREFILL.replace(T=512, E=4)
    d = gen.make_inputs(w)
    assert abs(d["x"].float().std().item() - w.sigma_x) < 0.02 * w.sigma_x
    assert abs(d["W_up"].float().std().item() - w.sigma_w) < 0.02 * w.sigma_w


# ------------------------------------------------------------------------------------------
# tile-aware sampling and the stage-by-stage checker, against a stand-in layer on the CPU
# ------------------------------------------------------------------------------------------

def test_gemm_tiles_cut_each_expert_segment_into_tiles():
    from oracle import oracle
    from parity import gemm_tiles
    ids = gen.make_topk_ids(300, 6, 2, seed=3, dist="skewed").numpy()
    al = oracle.align(ids, 6, 16)
    S = 600
    tiles = gemm_tiles(al["sorted_ids"], al["expert_ids"], al["num_post_padded"], S, 16, tile_m=128)
    flat = ids.reshape(-1)
    seen = np.concatenate(tiles)
    np.testing.assert_array_equal(np.sort(seen), np.arange(S))  # every slot once
    for tl in tiles:
        assert 1 <= tl.size <= 128 and np.all(flat[tl] == flat[tl[0]]) and np.all(np.diff(tl) > 0)
    counts = np.bincount(flat, minlength=6)
    assert len(tiles) == sum((c + 127) // 128 for c in counts)


def test_tile_sample_covers_first_and_last_row_of_every_tile():
    from parity import tile_sample
    rng = np.random.default_rng(0)
    tiles = [np.sort(rng.choice(4000, size=n, replace=False)) for n in (128, 128, 5, 1, 77)]
    tokens, slots, shared = tile_sample(tiles, T=1000, k=4, has_shared=True, min_tokens=300)
    for tl in tiles:
        assert tl[0] in slots and tl[-1] in slots
    assert {0, 127, 128, 255, 896, 999} <= set(shared.tolist())
    assert set((slots // 4).tolist()) <= set(tokens.tolist()) and tokens.size >= 300
    assert np.all(np.diff(tokens) > 0)


class _StandIn:
    """Plays the CUDA layer's part for check_stages: per-row results computed by the oracle and
    rounded the way the GPU stores them (h and y bf16, out fp32), laid out like the library's
    tile-ordered buffers."""

    def __init__(self, w, inp, res):
        from oracle import oracle
        T, k, E = w.T, w.top_k, w.E
        self.T, self.k = T, k
        kept = res["kept"].reshape(-1)
        slots = np.flatnonzero(kept)
        self.Mr = (slots.size + 127) // 128
        rows = self.Mr * 128 + ((T + 127) // 128) * 128
        ros = np.full(T * k, -1, dtype=np.int32)
        ros[slots] = np.arange(slots.size)
        tok = np.concatenate([slots // k, np.arange(T)])
        ex = np.concatenate([res["topk_ids"].reshape(-1)[slots], np.full(T, E)]).astype(np.int32)
        wts = np.concatenate([res["topk_w"].reshape(-1)[slots].astype(np.float32).astype(np.float64), np.ones(T)])
        r = np.concatenate([np.arange(slots.size), self.Mr * 128 + np.arange(T)])
        h = oracle.expert_h(inp["x"], inp, tok, ex)
        hb = torch.from_numpy(h).to(torch.bfloat16)
        y = oracle.expert_down(hb.double().numpy(), inp, ex, wts)
        ld = h.shape[1]
        self.h = torch.zeros((rows, ld), dtype=torch.bfloat16)
        self.y = torch.zeros((rows, w.H), dtype=torch.bfloat16)
        self.h[torch.as_tensor(r)] = hb
        self.y[torch.as_tensor(r)] = torch.from_numpy(y).to(torch.bfloat16)
        self.ros = torch.from_numpy(ros)
        out = np.zeros((T, w.H), dtype=np.float32)
        for t in range(T):
            acc = self.y[self.Mr * 128 + t].float().numpy().copy()
            for j in range(k):
                if ros[t * k + j] >= 0:
                    acc = acc + self.y[ros[t * k + j]].float().numpy()
            out[t] = acc
        self.out = torch.from_numpy(out)
        self.gw = res["topk_w"].astype(np.float32)

    def query(self, which):
        return 128

    def debug_expert_rows(self, T, k, device, with_h=True, stream=None):
        return {"h": self.h if with_h else None, "y": self.y, "row_of_slot": self.ros,
                "num_routed_tiles": torch.tensor([self.Mr], dtype=torch.int32)}


def _stage_setup():
    from oracle import oracle
    w = configs.MoEWorkload("stage_cpu", T=70, H=96, D=64, E=5, top_k=2, block_m=16, D_shared=32,
                            sigma_w=0.1, capacity_factor=1.0)
    inp = gen.make_inputs(w)
    res = oracle.forward(inp, w.top_k, w.block_m, w.capacity_factor)
    return w, inp, res, _StandIn(w, inp, res)


def _run_stages(w, inp, res, layer):
    from parity import check_stages, compact_weights
    T, k, E = w.T, w.top_k, w.E
    experts = np.arange(E)
    remap = np.arange(E + 1)
    cw = compact_weights(inp, experts)
    return check_stages(layer, w, inp, res["topk_ids"], layer.gw, layer.out, np.arange(T * k), np.arange(T),
                        np.arange(T), 128, cw, remap, inp["x"])


def test_stage_checker_accepts_values_rounded_like_the_gpu():
    w, inp, res, layer = _stage_setup()
    r = _run_stages(w, inp, res, layer)
    assert r["h_match"] == 1.0 and r["y_match"] == 1.0 and r["combine_err"] <= 1e-6


def _bump(t, row, col, ulps):
    """t[row, col] moved by `ulps` bf16 steps."""
    v = t[row, col].view(torch.int16)
    t[row, col] = (v + ulps).view(torch.bfloat16)


def test_stage_checker_rejects_planted_errors():
    import pytest
    w, inp, res, layer = _stage_setup()
    slot = int(np.flatnonzero(res["kept"].reshape(-1))[7])
    row = int(layer.ros[slot])
    # h three bf16 steps off in one element of one row
    _bump(layer.h, row, 5, 3)
    with pytest.raises(AssertionError, match="GEMM1"):
        _run_stages(w, inp, res, layer)
    _bump(layer.h, row, 5, -3)
    # y of one slot without its router weight
    saved = layer.y[row].clone()
    layer.y[row] = (layer.y[row].double() / float(layer.gw.reshape(-1)[slot])).to(torch.bfloat16)
    with pytest.raises(AssertionError, match="GEMM2"):
        _run_stages(w, inp, res, layer)
    layer.y[row] = saved
    # out of one token missing its shared-expert row
    t = 3
    layer.out[t] -= layer.y[layer.Mr * 128 + t].float()
    with pytest.raises(AssertionError, match="combine"):
        _run_stages(w, inp, res, layer)


# ------------------------------------------------------------------------------------------
# MXFP8: certified h-code flips
# ------------------------------------------------------------------------------------------

def test_mx_flip_steps_mark_only_elements_near_a_rounding_midpoint():
    from parity import mx_flip_steps
    # one block whose maximum is 3 (scale 2^(1-8) = 2^-7): value / scale = 128 * h
    h = np.zeros((1, 32))
    h[0, 0] = 230.4 / 128.0     # between the codes 224 and 240, 1.6 from their midpoint
    h[0, 1] = 3.0               # the maximum (code 384)
    h[0, 2] = 232.0 / 128.0     # exactly the midpoint of 224 and 240 (spacing 16)
    slack = np.full((1, 32), 1e-6)
    st = mx_flip_steps(h, slack)
    assert st[0, 2] == 16.0 / 128.0   # one E4M3 step, in h units
    assert st[0, 0] == 0.0 and st[0, 1] == 0.0 and np.count_nonzero(st) == 1
    # a block maximum within its slack of a power of two: the whole block is uncertain
    h2 = h.copy()
    h2[0, 1] = 4.0 * (1 - 1e-9)
    st2 = mx_flip_steps(h2, slack)
    assert np.all(st2[0, :3] > 0) and st2[0, 1] >= 4.0 / 8 * (1 - 1e-9)


def test_mx_certification_rejects_an_unexplained_error():
    import pytest
    from oracle import oracle
    from parity import certify_mx_flips, compact_weights
    w = configs.MoEWorkload("mx_cert", T=40, H=64, D=64, E=4, top_k=2, block_m=16, D_shared=32, sigma_w=0.1)
    inp = gen.make_inputs(w)
    res = oracle.forward(inp, w.top_k, w.block_m, mxfp8=True)
    tok = np.arange(w.T)
    cw = compact_weights(inp, np.arange(w.E))
    g_out = res["out"].copy()
    g_out[5, 7] += 0.05 * np.abs(res["out"]).max()  # 5% off in one element, no flip explains it
    with pytest.raises(AssertionError, match="exceed the tolerance"):
        certify_mx_flips(inp["x"], cw, tok, res["topk_ids"], res["topk_w"], res["kept"], g_out, res["out"], 1e-2, w)
    g_out[5, 7] = res["out"][5, 7]
    for t in range(3):  # too many tokens over the tolerance at all
        g_out[t, 0] += 0.05 * np.abs(res["out"]).max()
    with pytest.raises(AssertionError, match="over the tolerance"):
        certify_mx_flips(inp["x"], cw, tok, res["topk_ids"], res["topk_w"], res["kept"], g_out, res["out"], 1e-2, w)
