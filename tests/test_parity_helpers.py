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
