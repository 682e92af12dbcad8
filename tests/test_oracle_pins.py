"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU needed).

Each check uses a route that is independent of the oracle's code: hand-worked closed forms
(tests/golden), library routines (numpy/torch matmul, stable argsort), special cases that
reduce to a textbook FFN, invariances of the layer equation, and a dense brute force.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from mixture_experts_layer_block_b200 import configs, inputs as gen
from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def _f64(t):
    return t.to(torch.float64).numpy()


def _closed_form(expr):
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    s2 = 1.0 / (1.0 + math.exp(-2.0))
    return float(eval(expr, {"__builtins__": {}}, {"s1": s1, "s2": s2}))


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        fx = json.load(f)
    inp = {k: _bf16(fx[k]) for k in ("x", "W_router", "W_up", "W_gate", "W_down")}
    for k in ("Ws_up", "Ws_gate", "Ws_down"):
        inp[k] = _bf16(fx[k]) if k in fx else None
    inp["bias"] = None
    return fx, inp


# ----------------------------------------------------------------------------------------
# hand-worked examples (closed forms derived by hand, see the fixtures' derivation text)
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["hand_worked_layer.json", "hand_worked_capacity.json"])
def test_hand_worked_golden(name):
    fx, inp = _load(name)
    ex = fx["expect"]
    k = fx["top_k"]
    res = oracle.forward(inp, k, block_m=2, capacity_factor=fx["capacity_factor"])
    if "logits" in ex:
        np.testing.assert_array_equal(res["logits"], np.array(ex["logits"], dtype=np.float64))
    np.testing.assert_array_equal(res["topk_ids"], np.array(ex["topk_ids"]))
    w_exp = np.array([[_closed_form(e) for e in row] for row in ex["topk_w"]])
    np.testing.assert_allclose(res["topk_w"], w_exp, rtol=1e-15, atol=1e-15)
    out_exp = np.array([[_closed_form(e) for e in row] for row in ex["out"]])
    np.testing.assert_allclose(res["out"], out_exp, rtol=1e-14, atol=1e-15)
    if "kept" in ex:
        np.testing.assert_array_equal(res["kept"], np.array(ex["kept"]))
        assert res["capacity"] == ex["capacity"]
    for bm, al in ex["align"].items():
        r = oracle.align(res["topk_ids"], fx["E"], int(bm),
                         oracle.capacity(fx["T"], k, fx["E"], fx["capacity_factor"]))
        np.testing.assert_array_equal(r["sorted_ids"], al["sorted_ids"])
        np.testing.assert_array_equal(r["expert_ids"], al["expert_ids"])
        assert r["num_post_padded"] == al["num_post_padded"]


def test_silu_side_is_pinned():
    """A SiLU on the gate side (the common convention) must fail the hand-worked example."""
    fx, inp = _load("hand_worked_layer.json")
    swapped = dict(inp, W_up=inp["W_gate"], W_gate=inp["W_up"],
                   Ws_up=inp["Ws_gate"], Ws_gate=inp["Ws_up"])
    res = oracle.forward(swapped, fx["top_k"], block_m=2)
    out_exp = np.array([[_closed_form(e) for e in row] for row in fx["expect"]["out"]])
    assert np.max(np.abs(res["out"] - out_exp)) > 0.1


# ----------------------------------------------------------------------------------------
# stage pins against library routines
# ----------------------------------------------------------------------------------------

def test_router_logits_match_matmul():
    T, H, E = 37, 96, 11
    x = (torch.randn(T, H, generator=torch.Generator().manual_seed(1))).to(torch.bfloat16)
    w = (0.05 * torch.randn(E, H, generator=torch.Generator().manual_seed(2))).to(torch.bfloat16)
    bias = torch.randn(E, generator=torch.Generator().manual_seed(3))
    L, A = oracle.router_logits(x, w, bias.numpy(), with_absdot=True)
    ref = _f64(x) @ _f64(w).T + bias.double().numpy()
    np.testing.assert_allclose(L, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(A, np.abs(_f64(x)) @ np.abs(_f64(w)).T, rtol=1e-12, atol=1e-12)


def _topk_by_sort(L, k):
    """Definition by a stable lexicographic sort: value descending, index ascending."""
    T, E = L.shape
    ids = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(E), -L[t]))
        ids[t] = order[:k]
    p = np.exp(L - L.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, ids, axis=1)
    return ids, sel / sel.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("E,k,ties", [(8, 2, False), (64, 2, True), (256, 8, False),
                                      (256, 8, True), (5, 5, False), (7, 1, True)])
def test_topk_softmax_matches_sort_definition(E, k, ties):
    L = gen.make_logits(50, E, seed=E + k, ties=ties).double().numpy()
    ids, w = oracle.topk_softmax(L, k)
    ids_ref, w_ref = _topk_by_sort(L, k)
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_allclose(w, w_ref, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)


def test_topk_exact_ties_prefer_lower_index():
    L = np.zeros((1, 6))
    ids, w = oracle.topk_softmax(L, 3)
    np.testing.assert_array_equal(ids[0], [0, 1, 2])
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-15)


def _align_by_argsort(ids, E, bm, cap):
    """Align from a stable argsort of the flattened expert ids (a different route)."""
    flat = ids.reshape(-1).astype(np.int64)
    S = flat.size
    order = np.argsort(flat, kind="stable")
    kept = np.ones(S, dtype=bool)
    segs = []
    for e in range(E):
        slots = order[flat[order] == e]
        if cap > 0:
            kept[slots[cap:]] = False
            slots = slots[:cap]
        pad = -(-slots.size // bm) * bm
        segs.append(np.concatenate([slots, np.full(pad - slots.size, S)]).astype(np.int32))
    body = np.concatenate(segs) if segs else np.zeros(0, np.int32)
    L = S + E * (bm - 1)
    sorted_ids = np.full(L, S, dtype=np.int32)
    sorted_ids[:body.size] = body
    nb = -(-L // bm)
    expert_ids = np.full(nb, -1, dtype=np.int32)
    b = 0
    for e in range(E):
        nblk = segs[e].size // bm
        expert_ids[b:b + nblk] = e
        b += nblk
    return sorted_ids, expert_ids, body.size, kept.reshape(ids.shape)


def check_align_invariants(sorted_ids, expert_ids, P, ids, E, bm, kept):
    """Invariants that hold for any correct align output."""
    S = ids.size
    flat = ids.reshape(-1)
    assert P % bm == 0
    body = sorted_ids[:P]
    real = body[body != S]
    assert np.all(sorted_ids[P:] == S)
    # a permutation of the kept slot ids
    np.testing.assert_array_equal(np.sort(real), np.flatnonzero(kept.reshape(-1)))
    nb = P // bm
    eb = expert_ids[:nb]
    assert np.all(np.diff(eb) >= 0)          # non-decreasing
    assert np.all(expert_ids[nb:] == -1)
    for b in range(nb):
        blk = body[b * bm:(b + 1) * bm]
        r = blk[blk != S]
        assert r.size > 0                    # no block is all padding
        assert np.all(flat[r] == eb[b])      # every real id in block b belongs to its expert
        assert np.all(np.diff(r) > 0)        # ascending slot order inside the block
    counts = np.bincount(flat[kept.reshape(-1)], minlength=E)
    # every expert with tokens has ceil(n/bm) blocks, empty experts none
    nblk = np.bincount(eb, minlength=E)
    np.testing.assert_array_equal(nblk, -(-counts // bm))


@pytest.mark.parametrize("dist", ["random", "alternating_empty", "skewed", "one_expert"])
@pytest.mark.parametrize("bm", [16, 48, 128])
@pytest.mark.parametrize("cf", [0.0, 1.0])
def test_align_matches_argsort_definition(dist, bm, cf):
    T, E, k = 203, 32, 4
    ids = gen.make_topk_ids(T, E, k, seed=7, dist=dist).numpy()
    cap = oracle.capacity(T, k, E, cf)
    r = oracle.align(ids, E, bm, cap)
    s_ref, e_ref, P_ref, kept_ref = _align_by_argsort(ids, E, bm, cap)
    np.testing.assert_array_equal(r["sorted_ids"], s_ref)
    np.testing.assert_array_equal(r["expert_ids"], e_ref)
    assert r["num_post_padded"] == P_ref
    np.testing.assert_array_equal(r["kept"], kept_ref)
    check_align_invariants(r["sorted_ids"], r["expert_ids"], r["num_post_padded"], ids, E, bm, r["kept"])


def test_align_empty_input():
    ids = np.zeros((0, 2), dtype=np.int32)
    r = oracle.align(ids, 8, 16)
    assert r["num_post_padded"] == 0
    assert np.all(r["sorted_ids"] == 0)  # sentinel S = 0
    assert np.all(r["expert_ids"] == -1)


def test_capacity_keeps_first_slots_in_token_order():
    # 10 tokens all picking expert 3 first, E=4, k=2, cf=1 -> C = ceil(20/4) = 5
    ids = np.stack([np.full(10, 3), np.arange(10) % 3], axis=1).astype(np.int32)
    cap = oracle.capacity(10, 2, 4, 1.0)
    assert cap == 5
    r = oracle.align(ids, 4, 16, cap)
    kept = r["kept"]
    assert kept[:5, 0].all() and not kept[5:, 0].any()
    assert kept[:, 1].all()


# ----------------------------------------------------------------------------------------
# layer-equation pins: special cases, invariances, brute force
# ----------------------------------------------------------------------------------------

def _small_inputs(T=24, H=64, D=32, E=6, Ds=0, seed=0, sigma_w=0.1):
    w = configs.MoEWorkload("t", T=T, H=H, D=D, E=E, top_k=2, block_m=16, D_shared=Ds,
                            sigma_w=sigma_w, sigma_router=0.1, seed=seed)
    return w, gen.make_inputs(w)


def _ffn_torch(x, wu, wg, wd):
    """Textbook SwiGLU FFN with torch fp64 matmuls: W_down (SiLU(W_up x) * W_gate x)."""
    u = x @ wu.T
    g = x @ wg.T
    return (torch.nn.functional.silu(u) * g) @ wd.T


def test_single_expert_top1_is_plain_swiglu_ffn():
    w, inp = _small_inputs(E=1)
    res = oracle.forward(inp, 1, 16)
    x = inp["x"].double()
    ref = _ffn_torch(x, inp["W_up"][0].double(), inp["W_gate"][0].double(), inp["W_down"][0].double())
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-11, atol=1e-13)
    assert np.all(res["topk_w"] == 1.0)


def test_top_k_equals_E_is_dense_softmax_mixture():
    w, inp = _small_inputs(E=5, Ds=16)
    res = oracle.forward(inp, 5, 16)
    x = inp["x"].double()
    L = x @ inp["W_router"].double().T
    p = torch.softmax(L, dim=1)
    ref = _ffn_torch(x, inp["Ws_up"].double(), inp["Ws_gate"].double(), inp["Ws_down"].double())
    for e in range(5):
        ref = ref + p[:, e:e + 1] * _ffn_torch(x, inp["W_up"][e].double(), inp["W_gate"][e].double(),
                                               inp["W_down"][e].double())
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-11, atol=1e-13)


# ----------------------------------------------------------------------------------------
# the expert FFN stage by stage (GEMM1 + SwiGLU, GEMM2 with the router weight, combine)
# ----------------------------------------------------------------------------------------

def _stage_case():
    w, inp = _small_inputs(T=20, H=64, D=32, E=5, Ds=48, seed=3)
    rng = np.random.default_rng(4)
    tokens = rng.integers(0, w.T, size=40)
    experts = rng.integers(0, w.E + 1, size=40).astype(np.int32)  # E = the shared expert
    return w, inp, tokens, experts


def test_expert_h_is_swiglu_of_two_matmuls():
    """GEMM1 + SwiGLU against torch fp64: SiLU(x W_up^T) * (x W_gate^T), SiLU on the up side;
    the shared expert's rows (expert E) hold Ds entries; the projections and their |W x| sums
    against plain and abs matmuls."""
    w, inp, tokens, experts = _stage_case()
    h, uo, go, au, ag = oracle.expert_h(inp["x"], inp, tokens, experts, with_parts=True)
    x = inp["x"].double()
    for i, (t, e) in enumerate(zip(tokens, experts)):
        wu = inp["Ws_up"] if e == w.E else inp["W_up"][e]
        wg = inp["Ws_gate"] if e == w.E else inp["W_gate"][e]
        u = x[t] @ wu.double().T
        g = x[t] @ wg.double().T
        n = u.shape[0]
        np.testing.assert_allclose(h[i, :n], (torch.nn.functional.silu(u) * g).numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(uo[i, :n], u.numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(go[i, :n], g.numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(au[i, :n], (x[t].abs() @ wu.double().abs().T).numpy(), rtol=1e-12)
        np.testing.assert_allclose(ag[i, :n], (x[t].abs() @ wg.double().abs().T).numpy(), rtol=1e-12)


def test_expert_down_is_weighted_matmul():
    """GEMM2 against numpy fp64: wts[i] * W_down^e a[i] (W_down is [H][D]: out row c, in d)."""
    w, inp, tokens, experts = _stage_case()
    rng = np.random.default_rng(5)
    a = rng.standard_normal((tokens.size, max(w.D, w.D_shared)))
    wts = rng.uniform(-1.0, 1.0, size=tokens.size)
    y, ay = oracle.expert_down(a, inp, experts, wts, with_absdot=True)
    for i, e in enumerate(experts):
        wd = _f64(inp["Ws_down"] if e == w.E else inp["W_down"][e])
        n = wd.shape[1]
        np.testing.assert_allclose(y[i], wts[i] * (wd @ a[i, :n]), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(ay[i], abs(wts[i]) * (np.abs(wd) @ np.abs(a[i, :n])), rtol=1e-12)


def test_combine_sums_listed_rows_in_order():
    rng = np.random.default_rng(6)
    rows = rng.standard_normal((30, 17))
    idx = rng.integers(-1, 30, size=(9, 5))
    out = oracle.combine(rows, idx)
    for i in range(idx.shape[0]):
        ref = np.zeros(17)
        for r in idx[i]:
            if r >= 0:
                ref = ref + rows[r]
        np.testing.assert_array_equal(out[i], ref)


def test_stages_compose_to_the_layer():
    """Shared row, then the kept slots' weighted rows in j order, through the three stage
    functions, give the layer's output (capacity drops included)."""
    w, inp = _small_inputs(T=40, H=64, D=32, E=4, Ds=24, seed=7)
    res = oracle.forward(inp, 2, 16, capacity_factor=1.0)
    T, k = res["topk_ids"].shape
    tok = np.repeat(np.arange(T), k + 1)
    ex = np.concatenate([np.full((T, 1), w.E), res["topk_ids"]], axis=1).reshape(-1).astype(np.int32)
    wts = np.concatenate([np.ones((T, 1)), res["topk_w"]], axis=1).reshape(-1)
    h = oracle.expert_h(inp["x"], inp, tok, ex)
    y = oracle.expert_down(h, inp, ex, wts)
    keep = np.concatenate([np.ones((T, 1), dtype=bool), res["kept"]], axis=1)
    idx = np.where(keep, np.arange(T * (k + 1)).reshape(T, k + 1), -1)
    assert not keep.all()  # the case has capacity drops
    np.testing.assert_allclose(oracle.combine(y, idx), res["out"], rtol=1e-13, atol=1e-15)


def _brute_force(inp, k, cap_factor=0.0):
    """Dense per-token loop: every expert's FFN for every token, then the top-k sum.
    No sort of slots and no align; capacity applied by counting in token order."""
    x = _f64(inp["x"])
    T, H = x.shape
    wr = _f64(inp["W_router"])
    E = wr.shape[0]
    L = x @ wr.T
    if inp.get("bias") is not None:
        L = L + inp["bias"].double().numpy()
    wu, wg, wd = (_f64(inp[n]) for n in ("W_up", "W_gate", "W_down"))
    cap = math.ceil(cap_factor * T * k / E) if cap_factor > 0 else None
    used = [0] * E
    out = np.zeros((T, H))
    for t in range(T):
        ys = []
        for e in range(E):
            u = wu[e] @ x[t]
            g = wg[e] @ x[t]
            a = u / (1.0 + np.exp(-u)) * g
            ys.append(wd[e] @ a)
        order = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        p = np.exp(L[t] - L[t].max())
        p = p / p.sum()
        wsum = sum(p[e] for e in order)
        if inp.get("Ws_up") is not None:
            su, sg, sd = (_f64(inp[n]) for n in ("Ws_up", "Ws_gate", "Ws_down"))
            u = su @ x[t]
            g = sg @ x[t]
            out[t] += sd @ (u / (1.0 + np.exp(-u)) * g)
        for e in order:
            if cap is not None:
                used[e] += 1
                if used[e] > cap:
                    continue
            out[t] += (p[e] / wsum) * ys[e]
    return out


def test_brute_force_tiny_workload():
    w = configs.TINY
    inp = gen.make_inputs(w)
    res = oracle.forward(inp, w.top_k, w.block_m)
    ref = _brute_force(inp, w.top_k)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-11, atol=1e-12)


def test_brute_force_with_capacity_and_shared():
    w, inp = _small_inputs(T=40, E=4, Ds=8, seed=3)
    res = oracle.forward(inp, 2, 16, capacity_factor=0.6)
    assert res["kept"].sum() < res["kept"].size  # some slots dropped
    ref = _brute_force(inp, 2, cap_factor=0.6)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-11, atol=1e-12)


def test_brute_force_with_bias():
    w = configs.DECODE.replace(T=8, H=64, D=32, E=16, top_k=4)
    inp = gen.make_inputs(w)
    res = oracle.forward(inp, w.top_k, w.block_m)
    ref = _brute_force(inp, w.top_k)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-11, atol=1e-12)


def test_zero_down_projection_leaves_shared_only():
    w, inp = _small_inputs(Ds=16)
    z = dict(inp, W_down=torch.zeros_like(inp["W_down"]))
    res = oracle.forward(z, 2, 16)
    x = inp["x"].double()
    ref = _ffn_torch(x, inp["Ws_up"].double(), inp["Ws_gate"].double(), inp["Ws_down"].double())
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-11, atol=1e-13)


def test_zero_input_gives_zero_output():
    w, inp = _small_inputs(Ds=16)
    z = dict(inp, x=torch.zeros_like(inp["x"]))
    res = oracle.forward(z, 2, 16)
    assert np.all(res["out"] == 0.0)


def test_linear_in_down_projection():
    w, inp = _small_inputs()
    a = oracle.forward(inp, 2, 16)["out"]
    b = oracle.forward(dict(inp, W_down=(inp["W_down"].float() * 2).to(torch.bfloat16)), 2, 16)["out"]
    np.testing.assert_allclose(b, 2 * a, rtol=1e-13, atol=1e-15)


def test_expert_permutation_invariance():
    w, inp = _small_inputs(E=6)
    perm = torch.tensor([3, 0, 5, 1, 4, 2])
    q = dict(inp, W_router=inp["W_router"][perm], W_up=inp["W_up"][perm],
             W_gate=inp["W_gate"][perm], W_down=inp["W_down"][perm])
    a = oracle.forward(inp, 2, 16)
    b = oracle.forward(q, 2, 16)
    # away from ties the selected experts map through the permutation
    np.testing.assert_array_equal(perm.numpy()[b["topk_ids"]], a["topk_ids"])
    np.testing.assert_allclose(b["out"], a["out"], rtol=1e-12, atol=1e-14)


def test_token_permutation_equivariance():
    w, inp = _small_inputs(T=30)
    perm = torch.randperm(30, generator=torch.Generator().manual_seed(5))
    a = oracle.forward(inp, 2, 16)["out"]
    b = oracle.forward(dict(inp, x=inp["x"][perm]), 2, 16)["out"]
    np.testing.assert_allclose(b, a[perm.numpy()], rtol=1e-13, atol=1e-15)


def test_token_subset_matches_full_run():
    w, inp = _small_inputs(T=30, Ds=8)
    full = oracle.forward(inp, 2, 16)
    sub = oracle.layer(inp["x"], inp, full["topk_ids"], full["topk_w"], full["kept"], tokens=[29, 3, 17])
    np.testing.assert_array_equal(sub, full["out"][[29, 3, 17]])
