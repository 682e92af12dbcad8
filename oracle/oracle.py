"""Python face of the CPU oracle (moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()`` and by the
benchmark's CPU-baseline leg, never by the product package. It computes the layer forward in
IEEE double on bf16-valued inputs; see moe_oracle.c for the definitions and their sources.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (plain gcc, OpenMP, no host-specific ISA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(L):
    L.moe_oracle_router_logits.argtypes = [_p, _p, _p, _i64, _i64, _i64, _p, _p]
    L.moe_oracle_router_logits.restype = None
    L.moe_oracle_topk_softmax.argtypes = [_p, _i64, _i64, _i64, _p, _p]
    L.moe_oracle_topk_softmax.restype = None
    L.moe_oracle_align.argtypes = [_p, _i64, _i64, _i64, _i64, _i64, _p, _i64, _p, _i64, _p, _p]
    L.moe_oracle_align.restype = _i64
    L.moe_oracle_layer.argtypes = [_p, _i64, _i64, _i64, _i64, _i64, _p, _p, _p, _p, _p, _p,
                                   _i64, _p, _p, _p, _p, _i64, _p]
    L.moe_oracle_layer.restype = None
    L.moe_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    L.moe_oracle_e4m3_value.restype = ctypes.c_double
    L.moe_oracle_e4m3_encode.argtypes = [ctypes.c_double]
    L.moe_oracle_e4m3_encode.restype = ctypes.c_uint8
    L.moe_oracle_mx_quantize.argtypes = [_p, _i64, _p, _p]
    L.moe_oracle_mx_quantize.restype = None
    L.moe_oracle_mx_quantize_bf16_rows.argtypes = [_p, _i64, _i64, _p, _p]
    L.moe_oracle_mx_quantize_bf16_rows.restype = None
    L.moe_oracle_layer_mxfp8.argtypes = L.moe_oracle_layer.argtypes
    L.moe_oracle_layer_mxfp8.restype = None
    L.moe_oracle_expert_h.argtypes = [_p, _i64, _i64, _i64, _p, _p, _i64, _p, _p, _p, _p, _i64, _i64, _p,
                                      _p, _p, _p, _p]
    L.moe_oracle_expert_h.restype = None
    L.moe_oracle_expert_h_mxfp8.argtypes = L.moe_oracle_expert_h.argtypes
    L.moe_oracle_expert_h_mxfp8.restype = None
    L.moe_oracle_expert_down.argtypes = [_p, _i64, _i64, _i64, _i64, _p, _i64, _p, _p, _p, _i64, _p, _p]
    L.moe_oracle_expert_down.restype = None
    L.moe_oracle_combine.argtypes = [_p, _i64, _p, _i64, _i64, _p]
    L.moe_oracle_combine.restype = None
    L.moe_oracle_num_threads.argtypes = []
    L.moe_oracle_num_threads.restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def use_library(path: str | None):
    """Point this module at another build of moe_oracle.c (None = the default build).
    Used by the mutation test, which checks that planted mistakes fail the pins."""
    global _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))


def num_threads() -> int:
    return int(lib().moe_oracle_num_threads())


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def bf16_bits(t) -> np.ndarray:
    """Raw bf16 bit patterns (uint16, C-contiguous) of a torch bf16 tensor or of uint16 data."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch
    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------------------
# stages
# --------------------------------------------------------------------------------------

def router_logits(x, w_router, bias=None, with_absdot=False):
    xb, wb = bf16_bits(x), bf16_bits(w_router)
    T, H = xb.shape
    E = wb.shape[0]
    assert wb.shape == (E, H)
    b = None if bias is None else np.ascontiguousarray(np.asarray(bias, dtype=np.float32))
    logits = np.empty((T, E), dtype=np.float64)
    absdot = np.empty((T, E), dtype=np.float64) if with_absdot else None
    lib().moe_oracle_router_logits(_ptr(xb), _ptr(wb), _ptr(b), T, H, E, _ptr(logits), _ptr(absdot))
    return (logits, absdot) if with_absdot else logits


def topk_softmax(logits: np.ndarray, k: int):
    L = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = L.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    lib().moe_oracle_topk_softmax(_ptr(L), T, E, k, _ptr(ids), _ptr(w))
    return ids, w


def capacity(T: int, k: int, E: int, capacity_factor: float) -> int:
    """C = ceil(cf * T * k / E); 0 means dropless (cf <= 0)."""
    if capacity_factor <= 0:
        return 0
    return int(math.ceil(capacity_factor * T * k / E))


def max_sorted_len(T: int, k: int, E: int, block_m: int) -> int:
    return T * k + E * (block_m - 1)


def align(topk_ids: np.ndarray, E: int, block_m: int, cap: int = 0,
          sorted_len: int | None = None, blocks_len: int | None = None):
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, k = ids.shape
    if sorted_len is None:
        sorted_len = max_sorted_len(T, k, E, block_m)
    if blocks_len is None:
        blocks_len = (sorted_len + block_m - 1) // block_m
    sorted_ids = np.empty(sorted_len, dtype=np.int32)
    expert_ids = np.empty(blocks_len, dtype=np.int32)
    npp = np.zeros(1, dtype=np.int32)
    kept = np.empty(T * k, dtype=np.uint8)
    P = lib().moe_oracle_align(_ptr(ids), T, k, E, block_m, cap, _ptr(sorted_ids), sorted_len,
                               _ptr(expert_ids), blocks_len, _ptr(npp), _ptr(kept))
    if P < 0:
        raise ValueError("align output buffers too small")
    return {"sorted_ids": sorted_ids, "expert_ids": expert_ids, "num_post_padded": int(npp[0]),
            "kept": kept.reshape(T, k).astype(bool)}


def e4m3_value(code: int) -> float:
    """Value of an E4M3 code (NaN for S.1111.111)."""
    return float(lib().moe_oracle_e4m3_value(int(code)))


def e4m3_encode(v: float) -> int:
    """Nearest E4M3 code (ties to even, magnitudes above 448 clamped to 448)."""
    return int(lib().moe_oracle_e4m3_encode(float(v)))


def mx_quantize(v) -> tuple[np.ndarray, np.ndarray]:
    """MXFP8 (E4M3, 32-element blocks, E8M0 scales) of a float64 vector whose length is a
    multiple of 32: (codes uint8 [n], scale codes uint8 [n/32])."""
    a = np.ascontiguousarray(np.asarray(v, dtype=np.float64).ravel())
    assert a.size % 32 == 0
    codes = np.empty(a.size, dtype=np.uint8)
    scales = np.empty(a.size // 32, dtype=np.uint8)
    lib().moe_oracle_mx_quantize(_ptr(a), a.size, _ptr(codes), _ptr(scales))
    return codes, scales


def mx_values(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Values of MXFP8 data: E4M3 value of each code times 2^(scale code - 127) of its block."""
    c = np.asarray(codes, dtype=np.uint8).ravel()
    sc = np.repeat(np.asarray(scales, dtype=np.int64).ravel() - 127, 32)
    ev = np.array([e4m3_value(i) for i in range(256)], dtype=np.float64)
    return np.ldexp(ev[c], sc)


def mx_quantize_bf16_rows(m) -> tuple[np.ndarray, np.ndarray]:
    """MXFP8 of each row of a bf16 matrix [R][K] (K a multiple of 32): codes [R][K] and scale
    codes [R][K/32]."""
    b = bf16_bits(m)
    R, K = b.shape
    assert K % 32 == 0
    codes = np.empty((R, K), dtype=np.uint8)
    scales = np.empty((R, K // 32), dtype=np.uint8)
    lib().moe_oracle_mx_quantize_bf16_rows(_ptr(b), R, K, _ptr(codes), _ptr(scales))
    return codes, scales


def layer(x, weights: dict, topk_ids: np.ndarray, topk_w: np.ndarray, kept: np.ndarray,
          tokens=None, mxfp8: bool = False) -> np.ndarray:
    """Layer output rows (float64 [n, H]) for `tokens` (default: all). With `mxfp8`, x, h and
    every expert weight are MXFP8-quantised first (moe_oracle_layer_mxfp8)."""
    xb = bf16_bits(x)
    T, H = xb.shape
    wu, wg, wd = (bf16_bits(weights[n]) for n in ("W_up", "W_gate", "W_down"))
    E, D, H2 = wu.shape
    assert H2 == H and wd.shape == (E, H, D)
    k = topk_ids.shape[1]
    if weights.get("Ws_up") is not None:
        su, sg, sd = (bf16_bits(weights[n]) for n in ("Ws_up", "Ws_gate", "Ws_down"))
        Ds = su.shape[0]
    else:
        su = sg = sd = None
        Ds = 0
    tok = np.arange(T, dtype=np.int64) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int64)
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float64)
    kp = np.ascontiguousarray(kept, dtype=np.uint8)
    out = np.empty((tok.size, H), dtype=np.float64)
    fn = lib().moe_oracle_layer_mxfp8 if mxfp8 else lib().moe_oracle_layer
    if mxfp8:
        assert H % 32 == 0 and D % 32 == 0 and Ds % 32 == 0
    fn(_ptr(xb), T, H, D, E, k, _ptr(ids), _ptr(w), _ptr(kp), _ptr(wu), _ptr(wg), _ptr(wd), Ds, _ptr(su),
       _ptr(sg), _ptr(sd), _ptr(tok), tok.size, _ptr(out))
    return out


# --------------------------------------------------------------------------------------
# the expert FFN and the combine stage by stage (each stage can be fed another path's output
# of the stage before it)
# --------------------------------------------------------------------------------------

def _expert_mats(weights: dict):
    wu, wg, wd = (bf16_bits(weights[n]) for n in ("W_up", "W_gate", "W_down"))
    if weights.get("Ws_up") is not None:
        su, sg, sd = (bf16_bits(weights[n]) for n in ("Ws_up", "Ws_gate", "Ws_down"))
        Ds = su.shape[0]
    else:
        su = sg = sd = None
        Ds = 0
    return wu, wg, wd, su, sg, sd, Ds


def expert_h(x, weights: dict, tokens, experts, with_parts: bool = False, mxfp8: bool = False):
    """SwiGLU(W_up^e x_t, W_gate^e x_t) (float64 [n, max(D, Ds)]) for each (tokens[i],
    experts[i]); expert E (the number of routed experts) is the shared expert, whose rows hold
    Ds valid entries. With `with_parts` returns (h, u, g, au, ag): also the up and gate
    projections u = W_up x, g = W_gate x and their magnitude sums sum_h |W x|. With `mxfp8`, the
    MXFP8 layer's stage: x and the weight rows quantised, h rounded to fp32 (the values the layer
    then quantises)."""
    xb = bf16_bits(x)
    H = xb.shape[1]
    wu, wg, wd, su, sg, sd, Ds = _expert_mats(weights)
    E, D, _ = wu.shape
    tok = np.ascontiguousarray(tokens, dtype=np.int64)
    ex = np.ascontiguousarray(experts, dtype=np.int32)
    ld = max(D, Ds)
    h = np.zeros((tok.size, ld), dtype=np.float64)
    parts = [np.zeros_like(h) for _ in range(4)] if with_parts else [None] * 4
    fn = lib().moe_oracle_expert_h_mxfp8 if mxfp8 else lib().moe_oracle_expert_h
    fn(_ptr(xb), H, D, E, _ptr(wu), _ptr(wg), Ds, _ptr(su), _ptr(sg), _ptr(tok), _ptr(ex), tok.size, ld, _ptr(h),
       *(_ptr(q) for q in parts))
    return (h, *parts) if with_parts else h


def expert_down(a: np.ndarray, weights: dict, experts, wts, with_absdot: bool = False):
    """wts[i] * W_down^e a[i] (float64 [n, H]) with e = experts[i] (E = the shared expert); a is
    float64 [n, >= D (Ds)]. With `with_absdot` also |wts[i]| * sum_d |W_down^e a[i]|."""
    wu, wg, wd, su, sg, sd, Ds = _expert_mats(weights)
    E, H, D = wd.shape
    A = np.ascontiguousarray(a, dtype=np.float64)
    ex = np.ascontiguousarray(experts, dtype=np.int32)
    w = np.ascontiguousarray(wts, dtype=np.float64)
    y = np.empty((ex.size, H), dtype=np.float64)
    ay = np.empty_like(y) if with_absdot else None
    lib().moe_oracle_expert_down(_ptr(A), A.shape[1], H, D, E, _ptr(wd), Ds, _ptr(sd), _ptr(ex), _ptr(w), ex.size,
                                 _ptr(y), _ptr(ay))
    return (y, ay) if with_absdot else y


def combine(rows: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """out[i] = sum over j of rows[idx[i, j]] in j order, entries < 0 skipped (float64 [n, H])."""
    R = np.ascontiguousarray(rows, dtype=np.float64)
    I = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty((I.shape[0], R.shape[1]), dtype=np.float64)
    lib().moe_oracle_combine(_ptr(R), R.shape[1], _ptr(I), I.shape[0], I.shape[1], _ptr(out))
    return out


def forward(inputs: dict, top_k: int, block_m: int, capacity_factor: float = 0.0, tokens=None,
            mxfp8: bool = False):
    """Whole layer: router logits -> top-k softmax -> align (capacity) -> expert FFNs and the
    weighted combine for `tokens` (default all). Returns every intermediate. With `mxfp8` the
    expert FFNs run on MXFP8-quantised x, h and weights (the router stays bf16)."""
    logits, absdot = router_logits(inputs["x"], inputs["W_router"], inputs.get("bias"), with_absdot=True)
    T, E = logits.shape
    ids, w = topk_softmax(logits, top_k)
    cap = capacity(T, top_k, E, capacity_factor)
    al = align(ids, E, block_m, cap)
    out = layer(inputs["x"], inputs, ids, w, al["kept"], tokens, mxfp8=mxfp8)
    return {"logits": logits, "absdot": absdot, "topk_ids": ids, "topk_w": w, "capacity": cap,
            **al, "out": out}
