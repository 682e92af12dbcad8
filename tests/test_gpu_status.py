"""Device-side failure detection without a GPU fault: a bounded wait that runs out returns an
error status the host can read, and the context stays usable.

The stall is injected on the host: the down-projection tasks of one forward are told to wait
for more up-projection completions than exist, so their bounded dependency wait expires
after the configured (short) timeout.
"""
import pytest
import torch

from mixture_experts_layer_block_b200 import configs, inputs as gen
from parity import check_forward

pytestmark = pytest.mark.gpu


def test_injected_stall_reports_timeout_and_recovers():
    from mixture_experts_layer_block_b200.native import MOE_ERR_DEVICE_TIMEOUT, MoELayer
    w = configs.TINY
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = MoELayer.for_workload(w, timeout_ns=50_000_000)  # 50 ms
    out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
    layer.inject_stall(1)
    layer.forward(inp["x"], inp, out)
    rc, st = layer.status()
    assert rc == MOE_ERR_DEVICE_TIMEOUT
    assert st & (1 << 30)
    # status is cleared by the read and the next forward is correct
    assert layer.status() == (0, 0)
    check_forward(layer, w, inp)


def test_injected_stall_in_the_fused_small_batch_forward():
    """The same on a batch of at most 16 tokens, which runs as one fused launch: the down tasks'
    bounded wait runs out, no column block is combined, the status says so, and the next fused
    forward on the handle (its counters start afresh) is correct."""
    from mixture_experts_layer_block_b200.native import MOE_ERR_DEVICE_TIMEOUT, MoELayer
    w = configs.DSV3.replace(name="small_stall", T=12, H=512, D=256, E=16, top_k=4, D_shared=256)
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = MoELayer.for_workload(w, timeout_ns=50_000_000)
    out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
    layer.inject_stall(1)
    layer.forward(inp["x"], inp, out)
    assert layer.query(11) == 1
    rc, st = layer.status()
    assert rc == MOE_ERR_DEVICE_TIMEOUT and st & (1 << 30)
    assert layer.status() == (0, 0)
    check_forward(layer, w, inp)
    check_forward(layer, w, inp)


def test_invalid_arguments_are_rejected():
    from mixture_experts_layer_block_b200.native import (MOE_ERR_INVALID_ARG, MOE_ERR_MISALIGNED,
                                                         MoEError, MoELayer)
    w = configs.TINY
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = MoELayer.for_workload(w)
    out = torch.empty((w.T, w.H), dtype=torch.float32, device="cuda")
    with pytest.raises(MoEError) as e:
        layer.forward(inp["x"], inp, out, top_k=w.top_k + 1)
    assert e.value.code == MOE_ERR_INVALID_ARG
    big = torch.zeros((w.T + 1, w.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MoEError) as e:
        layer.forward(big, inp, torch.empty((w.T + 1, w.H), device="cuda"))
    assert e.value.code == MOE_ERR_INVALID_ARG
    raw = torch.zeros(w.T * w.H + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MoEError) as e:
        layer.forward(raw[1:1 + w.T * w.H].view(w.T, w.H), inp, out)
    assert e.value.code == MOE_ERR_MISALIGNED


@pytest.mark.parametrize("name,T,mx", [("dsv3_small", 300, False), ("small_fused", 12, False),
                                       ("dsv3_small_mx", 300, True), ("small_mx", 12, True)])
def test_trace_records_and_wait_accounting(name, T, mx):
    """MOE_FLAG_TRACE: one record per task (claimed by a CTA of the grid, finished after it was
    claimed), and per-CTA wait totals in which every wait fits inside its role's loop; the
    traced forward is still correct (bf16 and MXFP8 experts)."""
    import numpy as np
    from mixture_experts_layer_block_b200.native import MOE_FLAG_MXFP8, MOE_FLAG_TRACE, MoELayer
    w = configs.DSV3.replace(name=name, T=T, H=1024, D=256, E=32, D_shared=256)
    inp = {k: (v.cuda() if v is not None else None) for k, v in gen.make_inputs(w).items()}
    layer = MoELayer.for_workload(w, flags=MOE_FLAG_TRACE | (MOE_FLAG_MXFP8 if mx else 0))
    if mx:
        check_forward(layer, w, inp, wq=layer.quantize_experts_mxfp8(inp))
    else:
        check_forward(layer, w, inp)
    rec = layer.trace(1 << 16)
    tasks = layer.query(3)
    assert rec.shape[0] == tasks
    assert np.array_equal(np.sort(rec[:, 1]), np.arange(tasks))
    assert np.all((rec[:, 0] >= 0) & (rec[:, 0] < layer.query(1))) and np.all(rec[:, 3] >= rec[:, 2])
    waits = layer.trace_waits()
    assert waits.shape == (layer.query(0), len(MoELayer.WAITS))
    col = {n: waits[:, i] for i, n in enumerate(MoELayer.WAITS)}
    assert np.all(waits >= 0) and col["mma_loop"].sum() > 0 and col["epi_loop"].sum() > 0
    assert np.all(col["mma_full"] + col["mma_acc"] + col["mma_task"] <= col["mma_loop"])
    assert np.all(col["prod_empty"] + col["prod_dep"] + col["prod_ring"] + col["prod_claim"] <= col["prod_loop"])
    assert np.all(col["epi_task"] + col["epi_acc"] <= col["epi_loop"])
