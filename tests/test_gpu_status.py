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
