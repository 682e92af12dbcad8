"""The C-ABI library loads and exports every symbol include/moe_b200.h declares, and its host
checks reject bad arguments before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def native():
    from mixture_experts_layer_block_b200 import build
    build.build()
    from mixture_experts_layer_block_b200 import native
    return native


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API[^;(]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for required in ("moe_init", "moe_forward", "moe_destroy", "moe_get_status", "moe_debug_outputs",
                     "moe_gate_topk", "moe_align_block_size", "moe_router_logits"):
        assert required in names


def test_library_exports_every_declared_symbol(native):
    lib = ctypes.CDLL(native.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # and the binding knows each of them
    assert set(declared_symbols()) == set(native.SIGNATURES)


def _cfg(native, **kw):
    base = dict(hidden=256, inter=128, inter_shared=0, num_experts=8, top_k=2, block_m=16,
                capacity_factor=0.0, max_tokens=64, flags=0, device=-1, timeout_ns=0, claim_batch=0)
    base.update(kw)
    return native.moe_config(**base)


@pytest.mark.parametrize("bad", [dict(top_k=9), dict(top_k=0), dict(hidden=100), dict(inter=0),
                                 dict(num_experts=0), dict(num_experts=2048), dict(block_m=0),
                                 dict(max_tokens=0), dict(capacity_factor=-1.0),
                                 dict(inter_shared=12), dict(top_k=33, num_experts=64),
                                 dict(claim_batch=-1), dict(claim_batch=65)])
def test_init_rejects_bad_config_before_cuda(native, bad):
    h = ctypes.c_void_p()
    rc = native.lib.moe_init(ctypes.byref(_cfg(native, **bad)), ctypes.byref(h))
    assert rc == native.MOE_ERR_INVALID_ARG
    assert not h.value


def test_null_arguments(native):
    h = ctypes.c_void_p()
    assert native.lib.moe_init(None, ctypes.byref(h)) == native.MOE_ERR_INVALID_ARG
    assert native.lib.moe_forward(None, None, 0, None, None, None, None, None, None, 1, None, None) \
        == native.MOE_ERR_INVALID_ARG
    assert native.lib.moe_sorted_len(None, 4, 2) == -1
    assert native.lib.moe_debug_expert_rows(None, None, None, None, None, None) == native.MOE_ERR_INVALID_ARG
    native.lib.moe_destroy(None)


def test_status_strings(native):
    for code in range(-7, 1):
        assert native.lib.moe_status_string(code)


@pytest.mark.parametrize("bad", [dict(hidden=320), dict(inter=200), dict(inter_shared=64)])
def test_mxfp8_init_needs_multiples_of_128_before_cuda(native, bad):
    h = ctypes.c_void_p()
    rc = native.lib.moe_init(ctypes.byref(_cfg(native, flags=native.MOE_FLAG_MXFP8, **bad)), ctypes.byref(h))
    assert rc == native.MOE_ERR_UNSUPPORTED
    assert not h.value


def test_mxfp8_scale_bytes(native):
    f = native.lib.moe_mxfp8_scale_bytes
    assert f(128, 128) == 512
    assert f(7168, 2048) == 7168 * 2048 // 32
    for r, c in ((0, 128), (128, 0), (100, 128), (128, 96), (-128, 128)):
        assert f(r, c) == -1


def test_mxfp8_null_arguments(native):
    assert native.lib.moe_forward_mxfp8(None, None, 0, None, None, None, 1, None, None) == native.MOE_ERR_INVALID_ARG
    assert native.lib.moe_quantize_mxfp8(None, None, 128, 128, None, None, None) == native.MOE_ERR_INVALID_ARG


def test_binding_constants_match_the_header(native):
    """Every MOE_FLAG_* and MOE_ERR_* / MOE_OK value the header defines has the same value in
    the Python binding."""
    text = open(HEADER).read()
    defs = dict(re.findall(r"^#define\s+(MOE_(?:FLAG|ERR)_\w+|MOE_OK)\s+(-?\d+)u?\b", text, flags=re.M))
    assert len(defs) >= 15
    for name, value in defs.items():
        assert getattr(native, name) == int(value), name


def test_config_struct_matches_the_header(native):
    """moe_config's fields, in the header's order, with the C layout (int64 timeout_ns at 40,
    claim_batch after it, padded to 56 bytes)."""
    text = open(HEADER).read()
    body = re.search(r"typedef struct moe_config \{(.*?)\} moe_config;", text, flags=re.S).group(1)
    names = re.findall(r"^\s*(?:int32_t|uint32_t|int64_t|float)\s+(\w+);", body, flags=re.M)
    assert names == [f[0] for f in native.moe_config._fields_]
    assert native.moe_config.timeout_ns.offset == 40
    assert native.moe_config.claim_batch.offset == 48
    assert ctypes.sizeof(native.moe_config) == 56
