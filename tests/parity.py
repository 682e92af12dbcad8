"""Shared parity machinery: run the CUDA path and the oracle on the same seeded inputs and
compare them.

Routing is an integer decision taken on fp32 logits, so the GPU (tensor-core fp32
accumulation) and the oracle (fp64) may order two experts differently only when their
logits are closer than the rounding error of an fp32 dot product. Such tokens are accepted
only if the tie is certified (the oracle's gap is within the error bound
c * H * 2^-24 * sum_h |x_h w_h|) and they are left out of the element-wise output check;
every other token must match exactly in routing and within tolerance in value.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle

OUT_TOL = 1e-2      # max|gpu - ref| / max|ref| for bf16 tensor-core paths
STAGE_TOL = 1e-4    # fp32-accumulation stages compared stage by stage
ULP32 = 2.0 ** -24


def rel_err(a: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(a))) if a.size else 0.0
    return float(np.max(np.abs(a - ref)) / den)


def certified_routing(gpu_ids: np.ndarray, ref_logits: np.ndarray, absdot: np.ndarray, H: int,
                      safety: float = 4.0):
    """Per token: 0 = identical to the oracle's choice, 1 = different but every pick is
    within the fp32 error bound of the best remaining expert (a certified near-tie),
    2 = an uncertified difference."""
    T, k = gpu_ids.shape
    ref_ids, _ = oracle.topk_softmax(ref_logits, k)
    status = np.zeros(T, dtype=np.int8)
    bound = safety * H * ULP32 * absdot.max(axis=1) + 1e-30
    for t in np.flatnonzero(np.any(gpu_ids != ref_ids, axis=1)):
        v = ref_logits[t]
        remaining = np.ones(v.size, dtype=bool)
        ok = True
        for j in range(k):
            g = int(gpu_ids[t, j])
            if g < 0 or g >= v.size or not remaining[g]:
                ok = False
                break
            best = np.max(v[remaining])
            if v[g] < best - 2 * bound[t]:
                ok = False
                break
            remaining[g] = False
        status[t] = 1 if ok else 2
    return status, ref_ids


def gemm_tiles(sorted_ids: np.ndarray, expert_ids: np.ndarray, P: int, S: int, block_m: int,
               tile_m: int = 128) -> list:
    """The routed m-tiles of the expert GEMMs, each as the array of its slot ids in row order:
    each expert's segment of sorted_ids (its run of blocks in expert_ids) holds its kept slots
    first, then padding; the GEMMs cut those slots into tiles of tile_m rows."""
    tiles = []
    nb = P // block_m
    b = 0
    while b < nb:
        e = expert_ids[b]
        b1 = b
        while b1 < nb and expert_ids[b1] == e:
            b1 += 1
        seg = sorted_ids[b * block_m:b1 * block_m]
        seg = seg[seg < S]
        tiles += [seg[i:i + tile_m] for i in range(0, seg.size, tile_m)]
        b = b1
    return tiles


def tile_sample(tiles: list, T: int, k: int, has_shared: bool, tile_m: int = 128, min_tokens: int = 512,
                seed: int = 0):
    """Slots and tokens that cover every m-tile of the expert GEMMs: each routed tile gives its
    first row, its last row and one random row (so short tails, merged tails and the second tile
    of a group all appear), each shared-expert tile its first, last and one random token; random
    tokens are added up to `min_tokens`. Returns (tokens, slots, shared_tokens), sorted."""
    rng = np.random.default_rng(seed)
    slots = set()
    for tl in tiles:
        slots.update((int(tl[0]), int(tl[-1]), int(tl[rng.integers(tl.size)])))
    shared = set()
    if has_shared:
        for t0 in range(0, T, tile_m):
            t1 = min(T, t0 + tile_m)
            shared.update((t0, t1 - 1, int(rng.integers(t0, t1))))
    tokens = {s // k for s in slots} | shared
    if len(tokens) < min(min_tokens, T):
        rest = np.setdiff1d(np.arange(T), np.fromiter(tokens, dtype=np.int64))
        tokens |= set(rng.choice(rest, size=min(min_tokens, T) - len(tokens), replace=False).tolist())
    return (np.array(sorted(tokens), dtype=np.int64), np.array(sorted(slots), dtype=np.int64),
            np.array(sorted(shared), dtype=np.int64))


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    head = np.arange(min(n // 4, T))
    tail = np.arange(max(0, T - n // 4), T)
    mid = rng.choice(T, size=n - head.size - tail.size, replace=False)
    return np.unique(np.concatenate([head, tail, mid]))


def _kept_from_sorted(sorted_ids: np.ndarray, P: int, S: int) -> np.ndarray:
    kept = np.zeros(S, dtype=bool)
    body = sorted_ids[:P]
    kept[body[body < S]] = True
    return kept


def compact_weights(inp: dict, experts: np.ndarray) -> dict:
    """Host copies of just the listed experts' weights (the oracle needs no others)."""
    idx = torch.as_tensor(experts, dtype=torch.long, device=inp["W_up"].device)
    out = {n: inp[n].index_select(0, idx).cpu() for n in ("W_up", "W_gate", "W_down")}
    for n in ("Ws_up", "Ws_gate", "Ws_down"):
        out[n] = None if inp.get(n) is None else inp[n].cpu()
    return out


def check_forward(layer, w, inp: dict, tokens=None, out_tol: float = OUT_TOL, out_dtype=torch.float32,
                  wq: dict | None = None, stages: bool = True, min_tokens: int = 512):
    """Run the CUDA forward for workload `w` on `inp` (device tensors) and compare with the
    oracle on `tokens` (None = all; "tiles" = every m-tile's first, last and a random row, see
    tile_sample, topped up to `min_tokens`). With `wq` (the library's MXFP8 quantisation of the
    experts, from layer.quantize_experts_mxfp8) the MXFP8 forward runs instead, against the
    oracle's MXFP8 layer (which quantises the bf16 weights itself). With `stages` the expert
    GEMMs are also checked stage by stage (check_stages) on the same tiles' slots. Returns a
    dict of the measured errors and counts."""
    dev = inp["x"].device
    T, H, k, E = w.T, w.H, w.top_k, w.E
    out = torch.empty((T, H), dtype=out_dtype, device=dev)
    if wq is None:
        layer.forward(inp["x"], inp, out)
    else:
        layer.forward_mxfp8(inp["x"], inp["W_router"], inp.get("bias"), wq, out)
    dbg = layer.debug_outputs(T, k, dev)
    torch.cuda.synchronize()
    rc, st = layer.status()
    assert rc == 0 and st == 0, f"device status {rc} {st:#x}"

    # routing on the host: oracle logits in fp64 from the same bf16 inputs
    x_h = inp["x"].cpu()
    ref_logits, absdot = oracle.router_logits(x_h, inp["W_router"].cpu(),
                                              None if inp.get("bias") is None else inp["bias"].cpu().numpy(),
                                              with_absdot=True)
    g_logits = dbg["logits"].cpu().numpy().astype(np.float64)
    logit_err = rel_err(g_logits, ref_logits)
    g_ids = dbg["topk_ids"].cpu().numpy()
    status, ref_ids = certified_routing(g_ids, ref_logits, absdot, H)
    assert not np.any(status == 2), f"uncertified routing differences at tokens {np.flatnonzero(status == 2)[:10]}"
    _, ref_w = oracle.topk_softmax(ref_logits, k)

    cap = oracle.capacity(T, k, E, w.capacity_factor)
    ref_al = oracle.align(ref_ids, E, w.block_m, cap)
    g_sorted = dbg["sorted_ids"].cpu().numpy()
    g_expert = dbg["expert_ids"].cpu().numpy()
    g_P = int(dbg["num_post_padded"].cpu().item())
    n_tie = int(np.sum(status == 1))
    if n_tie == 0:
        # identical routing: the align outputs must be bit-exact
        np.testing.assert_array_equal(g_sorted, ref_al["sorted_ids"])
        np.testing.assert_array_equal(g_expert, ref_al["expert_ids"])
        assert g_P == ref_al["num_post_padded"]
    else:
        # still exact against the oracle's align of the GPU's own routing decisions
        own = oracle.align(g_ids, E, w.block_m, cap)
        np.testing.assert_array_equal(g_sorted, own["sorted_ids"])
        np.testing.assert_array_equal(g_expert, own["expert_ids"])
        assert g_P == own["num_post_padded"]
        assert n_tie <= max(2, T // 200), f"{n_tie} certified near-ties is implausibly many"
    g_kept = _kept_from_sorted(g_sorted, g_P, T * k).reshape(T, k)

    # which tokens to compare element-wise: same routing and same capacity decisions
    same = (status == 0) & np.all(g_kept == ref_al["kept"], axis=1)
    tile_m = layer.query(6)
    stage_slots = stage_shared = None
    if isinstance(tokens, str) and tokens == "tiles":
        tiles = gemm_tiles(g_sorted, g_expert, g_P, T * k, w.block_m, tile_m)
        tokens, stage_slots, stage_shared = tile_sample(tiles, T, k, w.D_shared > 0, tile_m, min_tokens)
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    if stage_slots is None:  # every slot and shared row of the compared tokens
        stage_slots = (tok[:, None] * k + np.arange(k)[None, :]).reshape(-1)
        stage_shared = tok if w.D_shared > 0 else np.zeros(0, dtype=np.int64)
    tok = tok[same[tok]]
    assert tok.size > 0
    w_err = float(np.max(np.abs(dbg["topk_w"].cpu().numpy()[same] - ref_w[same]))) if same.any() else 0.0

    # host copies of the weights of every expert the comparisons below need (once)
    sl_ids = g_ids.reshape(-1)[stage_slots] if stages else np.zeros(0, dtype=np.int32)
    experts = np.unique(np.concatenate([ref_ids[tok].reshape(-1), sl_ids]))
    remap = np.full(E + 1, -1, dtype=np.int64)
    remap[experts] = np.arange(experts.size)
    remap[E] = experts.size  # the shared expert, in the oracle's numbering
    cw = compact_weights(inp, experts)
    sub_ids = remap[ref_ids[tok]].astype(np.int32)
    ref_out = oracle.layer(x_h[torch.as_tensor(tok)], cw, sub_ids, ref_w[tok], ref_al["kept"][tok],
                           mxfp8=wq is not None)
    g_out = out.float().cpu().numpy()[tok].astype(np.float64)
    out_err = rel_err(g_out, ref_out)
    assert np.all(np.isfinite(g_out))
    res = {"logit_err": logit_err, "weight_err": w_err, "out_err": out_err, "near_ties": n_tie,
           "compared_tokens": int(tok.size), "P": g_P}
    assert logit_err <= STAGE_TOL, res
    assert w_err <= STAGE_TOL, res
    if wq is not None and out_err > out_tol:
        # MXFP8: tokens over the tolerance must owe the excess to h codes that may round either way
        res.update(certify_mx_flips(x_h, cw, tok, sub_ids, ref_w[tok], ref_al["kept"][tok], g_out, ref_out,
                                    out_tol, w))
    else:
        assert out_err <= out_tol, res
    if stages and out_dtype == torch.float32:
        res.update(check_stages(layer, w, inp, g_ids, dbg["topk_w"].cpu().numpy(), out, stage_slots,
                                stage_shared, tok, tile_m, cw, remap, x_h, gemm1=wq is None))
    return res


# ------------------------------------------------------------------------------------------
# MXFP8: certified h-code flips
# ------------------------------------------------------------------------------------------

def e4m3_spacing(v: np.ndarray) -> np.ndarray:
    """Spacing of the E4M3 values around |v| (2^-9 below 2^-6, else 2^(floor(log2 |v|) - 3))."""
    a = np.abs(v)
    sp = np.full(a.shape, 2.0 ** -9)
    big = a >= 2.0 ** -6
    sp[big] = 2.0 ** (np.floor(np.log2(a[big])) - 3)
    return sp


def mx_flip_steps(h: np.ndarray, slack: np.ndarray) -> np.ndarray:
    """For h (rows of fp32 values about to be MX-quantised in 32-element blocks) known only to
    within `slack` per element: the most the quantised value of each element can differ between
    two such evaluations -- 0 where the decision is certain; one E4M3 step where h lies within
    its slack of a rounding midpoint; for a block whose maximum lies within its slack of a power
    of two (the block scale may differ), an eighth of each element plus one subnormal step."""
    n, D = h.shape
    hb = h.reshape(n, D // 32, 32)
    sb = slack.reshape(n, D // 32, 32)
    amax = np.abs(hb).max(axis=2)
    smax = sb.max(axis=2)
    with np.errstate(divide="ignore"):
        e_lo = np.floor(np.log2(np.maximum(amax - smax, 1e-300)))
        e_hi = np.floor(np.log2(np.maximum(amax + smax, 1e-300)))
    scale = 2.0 ** (np.floor(np.log2(np.maximum(amax, 1e-300))) - 8)
    v = hb / scale[:, :, None]
    sp = e4m3_spacing(v)
    r = np.abs(v) / sp
    mid_dist = np.abs((r - np.floor(r)) - 0.5) * sp
    unsure = mid_dist <= sb / scale[:, :, None] + 1e-12 * sp
    steps = np.where(unsure, sp * scale[:, :, None], 0.0)
    scale_unsure = (e_lo != e_hi) & (amax > 0)
    wide = np.abs(hb) / 8.0 + 2.0 * 2.0 ** -9 * scale[:, :, None]
    steps = np.where(scale_unsure[:, :, None], wide, steps)
    return steps.reshape(n, D)


def certify_mx_flips(x_h, cw, tok, sub_ids, topk_w, kept, g_out, ref_out, out_tol, w):
    """The MXFP8 outputs of `tok` that exceed out_tol * max|ref|: each must be within that
    tolerance plus what its uncertain h codes can move it. Both sides quantise h from fp32
    values that differ by the two accumulation orders; where h sits within that difference of
    an E4M3 rounding midpoint (or the block maximum of a power of two), the codes may differ.
    The allowance is sum_j w_j sum_d |W_down^e_j[c][d]| * step_d (step from mx_flip_steps, the
    weights' own MX rounding bounded by a factor 1 + 2^-4). At most 1% of the tokens may need it."""
    den = float(np.max(np.abs(ref_out)))
    err = np.abs(g_out - ref_out)
    bad = np.flatnonzero(np.any(err > out_tol * den, axis=1))
    assert bad.size <= max(2, tok.size // 100), f"{bad.size} MXFP8 tokens over the tolerance"
    n_routed = cw["W_up"].shape[0]
    k = sub_ids.shape[1]
    t_rep, e_rep, w_rep, i_rep = [], [], [], []
    for i in bad:
        if cw.get("Ws_up") is not None:
            t_rep.append(int(tok[i])); e_rep.append(n_routed); w_rep.append(1.0); i_rep.append(i)
        for j in range(k):
            if kept[i, j]:
                t_rep.append(int(tok[i])); e_rep.append(int(sub_ids[i, j])); w_rep.append(float(topk_w[i, j]))
                i_rep.append(i)
    h, u, g, au, ag = oracle.expert_h(x_h, cw, np.array(t_rep), np.array(e_rep, dtype=np.int32), with_parts=True,
                                      mxfp8=True)
    du, dg = fp32_dot_slack(w.H, au), fp32_dot_slack(w.H, ag)
    sig = 1.0 / (1.0 + np.exp(-u))
    slack = 1.1 * (np.abs(g) * np.abs(sig * (1.0 + u * (1.0 - sig))) * du + np.abs(u * sig) * dg) \
        + 2.0 ** -19 * np.abs(h) + 2.0 ** -24 * np.abs(h)
    allow = np.zeros_like(g_out)
    n_unsure = 0
    for r in range(len(t_rep)):
        e = e_rep[r]
        wd = (cw["Ws_down"] if e == n_routed else cw["W_down"][e]).double().numpy()
        Dt = wd.shape[1]
        st = mx_flip_steps(h[r:r + 1, :Dt], slack[r:r + 1, :Dt])[0]
        n_unsure += int(np.count_nonzero(st))
        if st.any():
            allow[i_rep[r]] += abs(w_rep[r]) * (1.0 + 2.0 ** -4) * (np.abs(wd) @ st)
    ok = err[bad] <= out_tol * den + allow[bad]
    assert np.all(ok), (f"MXFP8 tokens {tok[bad][~np.all(ok, axis=1)][:5]} exceed the tolerance by more than "
                        f"their uncertain h codes allow")
    return {"mx_certified_tokens": int(bad.size), "mx_uncertain_h_codes": n_unsure,
            "out_err_after_allowance": float(np.max(np.maximum(err[bad] - allow[bad], 0.0)) / den)}


# ------------------------------------------------------------------------------------------
# stage-by-stage checks of the expert GEMMs and the combine
# ------------------------------------------------------------------------------------------

def bf16_round(v: np.ndarray) -> np.ndarray:
    """Values rounded to bf16 (nearest even), as float64."""
    return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float64)).to(torch.float32).to(
        torch.bfloat16).to(torch.float64).numpy()


def bf16_half_ulp(a: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at magnitude a (8 significant bits)."""
    a = np.maximum(np.abs(a), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def fp32_dot_slack(K: int, absdot: np.ndarray) -> np.ndarray:
    """Bound on the difference between an fp32-accumulated dot product of K bf16 products and
    its exact value: 8 sqrt(K) 2^-24 sum |terms| (rounding errors of random sign grow like
    sqrt(K); 8 is the margin)."""
    return 8.0 * np.sqrt(K) * ULP32 * absdot


def _check_rounded(name, gpu, ref, slack, min_match=0.95):
    """gpu (bf16 values) must be an fp32 value within `slack` of ref, rounded to bf16:
    |gpu - ref| <= slack + half a bf16 ulp at |ref| + slack; and most elements must equal ref
    rounded to bf16 exactly (the fp32 error rarely moves a value across a rounding boundary)."""
    bound = slack + bf16_half_ulp(np.abs(ref) + slack) + 1e-30
    bad = np.abs(gpu - ref) > bound
    assert not bad.any(), (f"{name}: {int(bad.sum())} elements outside the bound, e.g. gpu "
                           f"{gpu[bad][:4]} ref {ref[bad][:4]} bound {bound[bad][:4]}")
    match = float(np.mean(gpu == bf16_round(ref))) if gpu.size else 1.0
    assert match >= min_match, f"{name}: only {match:.3f} of the elements equal the oracle's value rounded"
    return match


def check_stages(layer, w, inp, g_ids, g_w, out, slots, shared_tokens, tokens, tile_m, cw, remap, x_h,
                 gemm1=True):
    """The layer equation's stages one by one, each fed the GPU's own output of the stage
    before it (so an error is caught in the stage that makes it):
      GEMM1 + SwiGLU  h of each slot (bf16) against the oracle's SwiGLU(W_up x, W_gate x),
      GEMM2           y = w_s W_down h of each slot (bf16), from the GPU's own h row,
      combine         out[t] (fp32) against the sum of the GPU's own y rows in slot order,
    on the listed slots (and the shared expert's rows of `shared_tokens`) and tokens. `cw` holds
    host copies of the needed experts' weights, `remap` maps expert ids (E = shared) into them.
    GEMM1 and GEMM2 are skipped for MXFP8 experts (h stays quantised); their combine is checked
    all the same."""
    dev = inp["x"].device
    T, k, E = w.T, w.top_k, w.E
    rows = layer.debug_expert_rows(T, k, dev, with_h=gemm1)
    if dev.type == "cuda":
        torch.cuda.synchronize()
    ros = rows["row_of_slot"].cpu().numpy()
    Mr = int(rows["num_routed_tiles"].item())
    ids_flat = g_ids.reshape(-1)
    sl = np.asarray(slots, dtype=np.int64)
    sl = sl[ros[sl] >= 0]
    sh = np.asarray(shared_tokens, dtype=np.int64)
    r_all = np.concatenate([ros[sl], (Mr + sh // tile_m) * tile_m + sh % tile_m]).astype(np.int64)
    tok_all = np.concatenate([sl // k, sh])
    ex_all = remap[np.concatenate([ids_flat[sl], np.full(sh.size, E)])].astype(np.int32)
    assert np.all(ex_all >= 0)
    n_routed = int(remap[E])
    w_all = np.concatenate([g_w.reshape(-1)[sl].astype(np.float64), np.ones(sh.size)])
    idx = torch.as_tensor(r_all, device=dev)
    res = {"stage_slots": int(sl.size), "stage_shared_rows": int(sh.size)}
    y_gpu = rows["y"].index_select(0, idx).double().cpu().numpy() if r_all.size else np.zeros((0, w.H))
    if gemm1 and r_all.size:
        Dt = np.where(ex_all == n_routed, w.D_shared, w.D)
        h_gpu = rows["h"].index_select(0, idx).double().cpu().numpy()
        h_ref, u, g, au, ag = oracle.expert_h(x_h, cw, tok_all, ex_all, with_parts=True)
        du, dg = fp32_dot_slack(w.H, au), fp32_dot_slack(w.H, ag)
        sig = 1.0 / (1.0 + np.exp(-u))
        dsilu = np.abs(sig * (1.0 + u * (1.0 - sig)))
        slack = 1.1 * (np.abs(g) * dsilu * du + np.abs(u * sig) * dg) + 2.0 ** -19 * np.abs(h_ref)
        cols = np.arange(h_ref.shape[1])[None, :] < Dt[:, None]
        res["h_match"] = _check_rounded("GEMM1+SwiGLU h", h_gpu[:, :h_ref.shape[1]][cols], h_ref[cols], slack[cols])
        # GEMM2 from the GPU's own h
        y_ref, ay = oracle.expert_down(h_gpu, cw, ex_all, w_all, with_absdot=True)
        slack_y = np.where((ex_all == n_routed)[:, None], fp32_dot_slack(max(w.D_shared, 1), ay),
                           fp32_dot_slack(w.D, ay)) + 2.0 ** -23 * np.abs(y_ref)
        res["y_match"] = _check_rounded("GEMM2 y", y_gpu, y_ref, slack_y)
    # combine from the GPU's own y rows: the shared row, then the kept slots in j order
    tk = np.asarray(tokens, dtype=np.int64)
    if tk.size:
        need = [(Mr + tk // tile_m) * tile_m + tk % tile_m] if w.D_shared > 0 else []
        need += [ros[tk * k + j] for j in range(k)]
        need = np.stack(need, axis=1).astype(np.int64)  # [n, (1) + k], -1 = dropped slot
        uniq, inv = np.unique(need[need >= 0], return_inverse=True)
        loc = np.full(need.shape, -1, dtype=np.int64)
        loc[need >= 0] = inv
        yr = rows["y"].index_select(0, torch.as_tensor(uniq, device=dev)).double().cpu().numpy()
        ref = oracle.combine(yr, loc)
        absum = oracle.combine(np.abs(yr), loc)
        got = out.float().cpu().numpy()[tk].astype(np.float64)
        bound = need.shape[1] * ULP32 * absum + 1e-30
        assert np.all(np.abs(got - ref) <= bound), "combine: fp32 sum outside its rounding bound"
        res["combine_err"] = rel_err(got, ref)
        assert res["combine_err"] <= STAGE_TOL, res
    return res
