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
                  wq: dict | None = None):
    """Run the CUDA forward for workload `w` on `inp` (device tensors) and compare with the
    oracle on `tokens` (None = all). With `wq` (the library's MXFP8 quantisation of the experts,
    from layer.quantize_experts_mxfp8) the MXFP8 forward runs instead, against the oracle's
    MXFP8 layer (which quantises the bf16 weights itself). Returns a dict of the measured errors
    and counts."""
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
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    tok = tok[same[tok]]
    assert tok.size > 0
    w_err = float(np.max(np.abs(dbg["topk_w"].cpu().numpy()[same] - ref_w[same]))) if same.any() else 0.0

    experts = np.unique(ref_ids[tok].reshape(-1))
    remap = np.full(E, -1, dtype=np.int64)
    remap[experts] = np.arange(experts.size)
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
    assert out_err <= out_tol, res
    return res
