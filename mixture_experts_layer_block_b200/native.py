"""ctypes binding of libmoe_b200.so (the C ABI in include/moe_b200.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels. The
functions keep the C names; ``MoELayer`` is a convenience owner of a handle that takes torch
tensors (device memory and streams come from PyTorch). There is no fallback: if the library
is missing this module raises on import.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_B200_LIBRARY may name another build of the same library (for A/B timing of builds)
LIB_PATH = os.environ.get("MOE_B200_LIBRARY") or os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_CUDA = -3
MOE_ERR_OUT_OF_MEMORY = -4
MOE_ERR_MISALIGNED = -5
MOE_ERR_DEVICE_TIMEOUT = -6
MOE_ERR_NOT_READY = -7

MOE_FLAG_STAGE_TIMING = 1
MOE_FLAG_HOST_STAGING = 2
MOE_FLAG_PAIR_TILES = 8
MOE_FLAG_SINGLE_TILES = 16
MOE_FLAG_OUT_BF16 = 32
MOE_FLAG_TAIL_TILES = 64
MOE_FLAG_NO_TAIL_TILES = 128
MOE_FLAG_STATIC_QUOTA = 256
MOE_FLAG_MXFP8 = 512
MOE_FLAG_UNFUSED_SMALL = 1024
MOE_FLAG_TWO_TILES = 2048
MOE_FLAG_TRACE = 4


class moe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("inter_shared", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("block_m", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("max_tokens", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("device", ctypes.c_int32),
                ("timeout_ns", ctypes.c_int64), ("claim_batch", ctypes.c_int32)]


class moe_shared_w(ctypes.Structure):
    _fields_ = [("up", ctypes.c_void_p), ("gate", ctypes.c_void_p), ("down", ctypes.c_void_p)]


class moe_mxfp8_mat(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class moe_mxfp8_experts(ctypes.Structure):
    _fields_ = [(n, moe_mxfp8_mat) for n in ("up", "gate", "down", "shared_up", "shared_gate", "shared_down")]


# every symbol the header declares, with its C signature
_P, _I32, _I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
SIGNATURES = {
    "moe_init": (ctypes.c_int, [ctypes.POINTER(moe_config), ctypes.POINTER(ctypes.c_void_p)]),
    "moe_destroy": (None, [_P]),
    "moe_forward": (ctypes.c_int, [_P, _P, _I32, _P, _P, _P, _P, _P, ctypes.POINTER(moe_shared_w),
                                   _I32, _P, _P]),
    "moe_forward_host": (ctypes.c_int, [_P, _P, _I32, _P, _P, _P, _P, _P,
                                        ctypes.POINTER(moe_shared_w), _I32, _P, _P]),
    "moe_forward_host_async": (ctypes.c_int, [_P, _P, _I32, _P, _P, _P, _P, _P,
                                              ctypes.POINTER(moe_shared_w), _I32, _P, _P]),
    "moe_forward_host_join": (ctypes.c_int, [_P, _P, _I32]),
    "moe_get_status": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32)]),
    "moe_mxfp8_scale_bytes": (_I64, [_I64, _I64]),
    "moe_quantize_mxfp8": (ctypes.c_int, [_P, _P, _I64, _I64, _P, _P, _P]),
    "moe_forward_mxfp8": (ctypes.c_int, [_P, _P, _I32, _P, _P, ctypes.POINTER(moe_mxfp8_experts), _I32, _P, _P]),
    "moe_router_logits": (ctypes.c_int, [_P, _P, _I32, _P, _P, _P, _P]),
    "moe_gate_topk": (ctypes.c_int, [_P, _P, _I32, _I32, _P, _P, _P]),
    "moe_align_block_size": (ctypes.c_int, [_P, _P, _I32, _I32, _P, _P, _P, _P]),
    "moe_sorted_len": (_I64, [_P, _I32, _I32]),
    "moe_blocks_len": (_I64, [_P, _I32, _I32]),
    "moe_debug_outputs": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_debug_expert_rows": (ctypes.c_int, [_P, _P, _P, _P, _P, _P]),
    "moe_stage_times": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_float), _I32]),
    "moe_query": (ctypes.c_int, [_P, _I32, ctypes.POINTER(ctypes.c_int64)]),
    "moe_trace_read": (ctypes.c_int, [_P, _P, _I64, ctypes.POINTER(ctypes.c_int64)]),
    "moe_debug_inject_stall": (ctypes.c_int, [_P, _I32]),
    "moe_trace_waits": (ctypes.c_int, [_P, _P, _I32, ctypes.POINTER(ctypes.c_int32)]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_align_block_size_noalloc": (ctypes.c_int, [_P, _I32, _I32, _I32, _I32, ctypes.c_float, _P, _P, _P,
                                                    _P]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_block_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def align_block_size_noalloc(topk_ids, num_experts, block_m, capacity_factor, sorted_ids, expert_ids,
                             num_post_padded, stream=None):
    """moe_align_block_size_noalloc on torch CUDA tensors (no handle, no allocation)."""
    T, k = topk_ids.shape
    check(lib.moe_align_block_size_noalloc(_ptr(topk_ids), T, k, num_experts, block_m, float(capacity_factor),
                                           _ptr(sorted_ids), _ptr(expert_ids), _ptr(num_post_padded),
                                           _stream(stream)), "moe_align_block_size_noalloc")


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {lib.moe_status_string(code).decode()} ({code})")
        self.code = code


def check(code: int, where: str) -> int:
    if code != MOE_OK:
        raise MoEError(code, where)
    return code


# ------------------------------------------------------------------------------------------
# torch-facing convenience (marshalling only)
# ------------------------------------------------------------------------------------------

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class MoELayer:
    """Owns one moe_handle. Tensors are torch CUDA tensors laid out as include/moe_b200.h
    states (x [T,H] bf16, W_router [E,H], W_up/W_gate [E,D,H], W_down [E,H,D] bf16, bias [E]
    fp32, out [T,H] fp32, or bf16 with MOE_FLAG_OUT_BF16)."""

    def __init__(self, hidden, inter, num_experts, top_k, block_m, max_tokens, inter_shared=0,
                 capacity_factor=0.0, flags=0, device=-1, timeout_ns=0, claim_batch=0):
        self.cfg = moe_config(hidden, inter, inter_shared, num_experts, top_k, block_m,
                              float(capacity_factor), max_tokens, flags, device, timeout_ns,
                              claim_batch)
        h = ctypes.c_void_p()
        check(lib.moe_init(ctypes.byref(self.cfg), ctypes.byref(h)), "moe_init")
        self.h = h
        self.out_dtype = "bfloat16" if flags & MOE_FLAG_OUT_BF16 else "float32"

    def _check_out(self, out):
        # the library writes out in the dtype the handle was configured for
        dt = getattr(out, "dtype", None)
        if dt is not None and str(dt).split(".")[-1] != self.out_dtype:
            raise TypeError(f"out must be {self.out_dtype} for this handle, got {dt}")

    @classmethod
    def for_workload(cls, w, max_tokens=None, **kw):
        return cls(w.H, w.D, w.E, w.top_k, w.block_m, max_tokens or w.T, inter_shared=w.D_shared,
                   capacity_factor=w.capacity_factor, **kw)

    def close(self):
        if getattr(self, "h", None):
            lib.moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _shared(self, wts):
        if wts.get("Ws_up") is None:
            return None
        s = moe_shared_w(wts["Ws_up"].data_ptr(), wts["Ws_gate"].data_ptr(), wts["Ws_down"].data_ptr())
        return ctypes.byref(s), s

    def forward(self, x, wts, out, top_k=None, stream=None):
        self._check_out(out)
        sh = self._shared(wts)
        check(lib.moe_forward(self.h, _ptr(x), x.shape[0], _ptr(wts["W_router"]), _ptr(wts.get("bias")),
                              _ptr(wts["W_up"]), _ptr(wts["W_gate"]), _ptr(wts["W_down"]),
                              sh[0] if sh else None, top_k or self.cfg.top_k, _ptr(out),
                              _stream(stream)), "moe_forward")
        return out

    def forward_host(self, x_host, wts, out_host, top_k=None, stream=None):
        self._check_out(out_host)
        sh = self._shared(wts)
        check(lib.moe_forward_host(self.h, _ptr(x_host), x_host.shape[0], _ptr(wts["W_router"]),
                                   _ptr(wts.get("bias")), _ptr(wts["W_up"]), _ptr(wts["W_gate"]),
                                   _ptr(wts["W_down"]), sh[0] if sh else None, top_k or self.cfg.top_k,
                                   _ptr(out_host), _stream(stream)), "moe_forward_host")
        return out_host

    def forward_host_async(self, x_host, wts, out_host, top_k=None, stream=None):
        """Queue a host-buffer forward; consecutive calls overlap their copies with the
        previous forward. x_host / out_host must stay alive until forward_host_join."""
        self._check_out(out_host)
        sh = self._shared(wts)
        check(lib.moe_forward_host_async(self.h, _ptr(x_host), x_host.shape[0], _ptr(wts["W_router"]),
                                         _ptr(wts.get("bias")), _ptr(wts["W_up"]), _ptr(wts["W_gate"]),
                                         _ptr(wts["W_down"]), sh[0] if sh else None,
                                         top_k or self.cfg.top_k, _ptr(out_host), _stream(stream)),
              "moe_forward_host_async")
        return out_host

    # ---- MXFP8 experts ----
    def quantize_mxfp8(self, src, stream=None):
        """MXFP8 of a bf16 CUDA matrix [R, K] (a 3-D tensor is viewed as [-1, K]): returns
        (codes uint8 [R, K], scales uint8 [R*K/32] in the header's atom layout)."""
        import torch
        m = src.reshape(-1, src.shape[-1])
        R, K = m.shape
        nb = lib.moe_mxfp8_scale_bytes(R, K)
        if nb < 0:
            raise ValueError(f"MXFP8 needs both dimensions multiples of 128, got {R}x{K}")
        q = torch.empty(R, K, dtype=torch.uint8, device=src.device)
        sf = torch.empty(nb, dtype=torch.uint8, device=src.device)
        check(lib.moe_quantize_mxfp8(self.h, _ptr(m), R, K, _ptr(q), _ptr(sf), _stream(stream)),
              "moe_quantize_mxfp8")
        return q, sf

    def quantize_experts_mxfp8(self, wts, stream=None):
        """The quantised experts of a weight dict (keys W_up, W_gate, W_down and, with a
        shared expert, Ws_up, Ws_gate, Ws_down) as {name: (codes, scales)}."""
        names = ["W_up", "W_gate", "W_down"] + (["Ws_up", "Ws_gate", "Ws_down"] if wts.get("Ws_up") is not None else [])
        return {n: self.quantize_mxfp8(wts[n], stream) for n in names}

    def forward_mxfp8(self, x, w_router, bias, wq, out, top_k=None, stream=None):
        """moe_forward_mxfp8: wq as returned by quantize_experts_mxfp8 (needs MOE_FLAG_MXFP8)."""
        self._check_out(out)
        mats = []
        for n in ("W_up", "W_gate", "W_down", "Ws_up", "Ws_gate", "Ws_down"):
            q, sf = wq.get(n, (None, None))
            mats.append(moe_mxfp8_mat(None if q is None else q.data_ptr(), None if sf is None else sf.data_ptr()))
        ex = moe_mxfp8_experts(*mats)
        check(lib.moe_forward_mxfp8(self.h, _ptr(x), x.shape[0], _ptr(w_router), _ptr(bias), ctypes.byref(ex),
                                    top_k or self.cfg.top_k, _ptr(out), _stream(stream)), "moe_forward_mxfp8")
        return out

    def forward_host_join(self, stream=None, block=True):
        check(lib.moe_forward_host_join(self.h, _stream(stream), 1 if block else 0), "moe_forward_host_join")

    def router_logits(self, x, w_router, bias, logits, stream=None):
        check(lib.moe_router_logits(self.h, _ptr(x), x.shape[0], _ptr(w_router), _ptr(bias), _ptr(logits),
                                    _stream(stream)), "moe_router_logits")
        return logits

    def gate_topk(self, logits, top_k, ids, w, stream=None):
        check(lib.moe_gate_topk(self.h, _ptr(logits), logits.shape[0], top_k, _ptr(ids), _ptr(w),
                                _stream(stream)), "moe_gate_topk")
        return ids, w

    def align(self, topk_ids, sorted_ids, expert_ids, npp, stream=None):
        T, k = topk_ids.shape
        check(lib.moe_align_block_size(self.h, _ptr(topk_ids), T, k, _ptr(sorted_ids), _ptr(expert_ids),
                                       _ptr(npp), _stream(stream)), "moe_align_block_size")

    def sorted_len(self, T, k):
        return int(lib.moe_sorted_len(self.h, T, k))

    def blocks_len(self, T, k):
        return int(lib.moe_blocks_len(self.h, T, k))

    def debug_outputs(self, T, k, device, stream=None):
        import torch
        E = self.cfg.num_experts
        d = {"logits": torch.empty((T, E), dtype=torch.float32, device=device),
             "topk_ids": torch.empty((T, k), dtype=torch.int32, device=device),
             "topk_w": torch.empty((T, k), dtype=torch.float32, device=device),
             "sorted_ids": torch.empty((self.sorted_len(T, k),), dtype=torch.int32, device=device),
             "expert_ids": torch.empty((self.blocks_len(T, k),), dtype=torch.int32, device=device),
             "num_post_padded": torch.empty((1,), dtype=torch.int32, device=device)}
        check(lib.moe_debug_outputs(self.h, *(_ptr(d[n]) for n in ("logits", "topk_ids", "topk_w",
                                                                    "sorted_ids", "expert_ids",
                                                                    "num_post_padded")),
                                    _stream(stream)), "moe_debug_outputs")
        return d

    def debug_expert_rows(self, T, k, device, with_h=True, stream=None):
        """moe_debug_expert_rows: the GEMM rows of the last forward, as torch tensors (h and y
        bf16 [rows, ...], row_of_slot int32 [T*k], num_routed_tiles int)."""
        import torch
        rows, ldh = self.query(9), self.query(10)
        d = {"h": torch.empty((rows, ldh), dtype=torch.bfloat16, device=device) if with_h else None,
             "y": torch.empty((rows, self.cfg.hidden), dtype=torch.bfloat16, device=device),
             "row_of_slot": torch.empty((T * k,), dtype=torch.int32, device=device),
             "num_routed_tiles": torch.empty((1,), dtype=torch.int32, device=device)}
        check(lib.moe_debug_expert_rows(self.h, _ptr(d["h"]), _ptr(d["y"]), _ptr(d["row_of_slot"]),
                                        _ptr(d["num_routed_tiles"]), _stream(stream)), "moe_debug_expert_rows")
        return d

    def status(self):
        st = ctypes.c_int32(0)
        rc = lib.moe_get_status(self.h, ctypes.byref(st))
        return rc, st.value

    STAGES = ("router", "gating", "align_scatter", "row_gather", "expert_gemm", "combine")

    def stage_times(self):
        ms = (ctypes.c_float * 6)()
        check(lib.moe_stage_times(self.h, ms, 6), "moe_stage_times")
        return list(ms)

    def query(self, which):
        v = ctypes.c_int64(0)
        check(lib.moe_query(self.h, which, ctypes.byref(v)), "moe_query")
        return v.value

    def trace(self, cap):
        import numpy as np
        buf = np.zeros((cap, 4), dtype=np.int64)
        n = ctypes.c_int64(0)
        check(lib.moe_trace_read(self.h, buf.ctypes.data_as(ctypes.c_void_p), cap, ctypes.byref(n)),
              "moe_trace_read")
        return buf[: n.value]

    WAITS = ("prod_empty", "prod_dep", "prod_ring", "prod_claim", "mma_full", "mma_acc", "mma_task",
             "epi_task", "epi_acc", "prod_loop", "mma_loop", "epi_loop", "front_router", "front_schedule",
             "front_gather", "front_last", "front_to_end", "sched_arrive", "sched_logits", "sched_gating",
             "sched_tables", "sched_writes", "sched_publish", "combine_count", "combine_run")

    def trace_waits(self):
        """moe_trace_waits: [CTAs, 25] int64 ns (columns named by WAITS)."""
        import numpy as np
        buf = np.zeros((1024, len(self.WAITS)), dtype=np.int64)
        n = ctypes.c_int32(0)
        check(lib.moe_trace_waits(self.h, buf.ctypes.data_as(ctypes.c_void_p), 1024, ctypes.byref(n)),
              "moe_trace_waits")
        return buf[: n.value]

    def inject_stall(self, extra):
        check(lib.moe_debug_inject_stall(self.h, extra), "moe_debug_inject_stall")
