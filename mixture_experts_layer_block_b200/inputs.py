"""Seeded synthetic inputs for the MoE layer.

This module holds only random-number drawing and the input recipe: no step of the layer is
computed here, so both the CUDA path and the CPU oracle may read what it produces.

Recipe: every tensor is drawn as fp32 ``randn * sigma`` from its own torch.Generator seeded
with ``1000 * seed + index`` (index order: x, W_router, W_up, W_gate, W_down, W_shared_up,
W_shared_gate, W_shared_down, router bias) and rounded to bf16. Large tensors are drawn
one expert at a time so that the fp32 temporaries stay small; the draw order is fixed, so a
given (workload, seed, device) always yields the same values. The CPU and CUDA generators
produce different streams, so a test that compares against the oracle draws on one device
and copies.

Layouts (all row-major, contiguous):
  x         [T, H]      bf16
  W_router  [E, H]      bf16   (output-major, like a Linear layer's weight)
  W_up      [E, D, H]   bf16
  W_gate    [E, D, H]   bf16
  W_down    [E, H, D]   bf16
  Ws_up     [Ds, H], Ws_gate [Ds, H], Ws_down [H, Ds]  bf16 (only when Ds > 0)
  bias      [E]         fp32 or None
"""
from __future__ import annotations

import math

import torch

from .configs import MoEWorkload

IDX_X, IDX_WR, IDX_WU, IDX_WG, IDX_WD, IDX_SU, IDX_SG, IDX_SD, IDX_BIAS = range(9)


def _gen(seed: int, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + index)
    return g


def _randn_bf16(shape, sigma, g, device, chunks=1):
    """fp32 N(0, sigma) rounded to bf16, drawn in `chunks` pieces along dim 0."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    n0 = shape[0]
    step = max(1, math.ceil(n0 / chunks))
    for s in range(0, n0, step):
        e = min(n0, s + step)
        tmp = torch.randn((e - s,) + tuple(shape[1:]), generator=g, device=device,
                          dtype=torch.float32)
        if sigma != 1.0:
            tmp.mul_(sigma)
        out[s:e].copy_(tmp)
        del tmp
    return out


def router_bias(w: MoEWorkload, device="cpu"):
    """Per-expert router-logit bias of the workload (fp32 [E]) or None."""
    if w.bias == "none":
        return None
    if w.bias == "gaussian":
        g = _gen(w.seed, IDX_BIAS, device)
        return torch.randn((w.E,), generator=g, device=device, dtype=torch.float32)
    if w.bias == "zipf":
        rank = torch.arange(1, w.E + 1, dtype=torch.float64)
        return (2.0 * torch.log(1.0 / rank)).to(torch.float32).to(device)
    raise ValueError(f"unknown bias kind {w.bias!r}")


def make_x(w: MoEWorkload, device="cpu", T: int | None = None) -> torch.Tensor:
    T = w.T if T is None else T
    return _randn_bf16((T, w.H), w.sigma_x, _gen(w.seed, IDX_X, device), device,
                       chunks=max(1, (T * w.H) // (1 << 26)))


def make_weights(w: MoEWorkload, device="cpu") -> dict:
    """All weights of the layer for workload `w` (see the module docstring for layouts)."""
    per_expert = w.E if w.E * w.D * w.H > (1 << 24) else 1
    out = {
        "W_router": _randn_bf16((w.E, w.H), w.sigma_router, _gen(w.seed, IDX_WR, device), device),
        "W_up": _randn_bf16((w.E, w.D, w.H), w.sigma_w, _gen(w.seed, IDX_WU, device), device,
                            chunks=per_expert),
        "W_gate": _randn_bf16((w.E, w.D, w.H), w.sigma_w, _gen(w.seed, IDX_WG, device), device,
                              chunks=per_expert),
        "W_down": _randn_bf16((w.E, w.H, w.D), w.sigma_w, _gen(w.seed, IDX_WD, device), device,
                              chunks=per_expert),
        "bias": router_bias(w, device),
    }
    if w.D_shared > 0:
        out["Ws_up"] = _randn_bf16((w.D_shared, w.H), w.sigma_w, _gen(w.seed, IDX_SU, device), device)
        out["Ws_gate"] = _randn_bf16((w.D_shared, w.H), w.sigma_w, _gen(w.seed, IDX_SG, device), device)
        out["Ws_down"] = _randn_bf16((w.H, w.D_shared), w.sigma_w, _gen(w.seed, IDX_SD, device), device)
    else:
        out["Ws_up"] = out["Ws_gate"] = out["Ws_down"] = None
    return out


def make_inputs(w: MoEWorkload, device="cpu") -> dict:
    d = make_weights(w, device)
    d["x"] = make_x(w, device)
    return d


# ---------------------------------------------------------------------------------------
# Synthetic routing and logits for the stage tests (gating and align take these as inputs)
# ---------------------------------------------------------------------------------------

def make_logits(T: int, E: int, seed: int, device="cpu", kind: str = "randn",
                ties: bool = False) -> torch.Tensor:
    """fp32 router logits [T, E]. kind: randn | zipf (randn plus -2*log(e+1)).
    With ties=True every value is rounded to a coarse grid so exact ties are frequent."""
    g = _gen(seed, 100, device)
    L = torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    if kind == "zipf":
        rank = torch.arange(1, E + 1, dtype=torch.float64)
        L = L + (2.0 * torch.log(1.0 / rank)).to(torch.float32).to(device)
    if ties:
        L = torch.round(L * 4.0) / 4.0
    return L


def make_topk_ids(T: int, E: int, k: int, seed: int, dist: str = "random",
                  device="cpu") -> torch.Tensor:
    """int32 expert ids [T, k], each row k distinct experts.

    dist: random          uniform over experts
          alternating_empty  only even experts receive tokens
          skewed          Zipf-like preference for low expert ids
          one_expert      every token's first choice is expert 0 (others uniform)
          empty           T rows of nothing (T should be 0)
    """
    g = _gen(seed, 200, device="cpu")
    if T == 0:
        return torch.zeros((0, k), dtype=torch.int32, device=device)
    if dist == "alternating_empty":
        pool = torch.arange(0, E, 2)
    else:
        pool = torch.arange(E)
    n = pool.numel()
    if k > n:
        raise ValueError("top_k larger than the experts that may receive tokens")
    if dist in ("random", "alternating_empty", "one_expert"):
        scores = torch.rand((T, n), generator=g)
        if dist == "one_expert":
            scores[:, 0] = 2.0
    elif dist == "skewed":
        scores = torch.rand((T, n), generator=g) / torch.arange(1, n + 1, dtype=torch.float32)
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    idx = torch.argsort(scores, dim=1, descending=True, stable=True)[:, :k]
    return pool[idx].to(torch.int32).to(device).contiguous()
