"""Pins of the oracle's MXFP8 arithmetic (no GPU needed).

The pages name MXFP8 experts without defining the format; the oracle reads it as the OCP
Microscaling format MXFP8 (E4M3 elements, 32-element blocks, E8M0 scales). These checks fix
that arithmetic by routes independent of the oracle's code: the E4M3 bit layout written out
by hand, torch's own float8_e4m3fn conversion, the scale rule's closed form, exact round trips
of data built on the MX grid, the rounding error bound, a hand-worked layer, and invariances of
the layer under power-of-two scalings.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


# ----------------------------------------------------------------------------------------
# E4M3 elements
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x30, 0.5),
    (0x38, 1.0), (0x39, 1.125), (0x3F, 1.875), (0x40, 2.0), (0x70, 128.0), (0x78, 256.0),
    (0x7E, 448.0), (0xB8, -1.0), (0xFE, -448.0), (0x81, -(2.0 ** -9)),
])
def test_e4m3_decode_table(code, value):
    """Sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 = subnormals."""
    assert oracle.e4m3_value(code) == value


def test_e4m3_nan_codes():
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))


def test_e4m3_every_finite_code_round_trips():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c, hex(c)


def test_e4m3_ties_go_to_the_even_code():
    for c in range(0x00, 0x7E):
        lo, hi = oracle.e4m3_value(c), oracle.e4m3_value(c + 1)
        mid = 0.5 * (lo + hi)
        even = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == even, hex(c)
        assert oracle.e4m3_encode(-mid) == 0x80 | even, hex(c)
        assert oracle.e4m3_encode(mid - (hi - lo) / 8) == c
        assert oracle.e4m3_encode(mid + (hi - lo) / 8) == c + 1


def test_e4m3_saturates_at_448():
    for v in (448.0, 449.0, 463.99, 464.0, 1e6, 1e300):
        assert oracle.e4m3_encode(v) == 0x7E
        assert oracle.e4m3_encode(-v) == 0xFE


def test_e4m3_matches_torch_float8_conversion():
    """torch's float32 -> float8_e4m3fn conversion rounds to nearest even; in range the two
    conversions must agree bit for bit."""
    g = torch.Generator().manual_seed(7)
    mags = torch.exp2(torch.empty(20000).uniform_(-12.0, 8.8, generator=g))
    v = (mags * torch.sign(torch.randn(20000, generator=g))).clamp(-448.0, 448.0).float()
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(a)) for a in v.numpy()], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


# ----------------------------------------------------------------------------------------
# MX blocks
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("j", [-20, -7, -1, 0, 1, 5, 8, 15])
@pytest.mark.parametrize("pos", [0, 13, 31])
def test_scale_code_is_floor_log2_amax_minus_8(j, pos):
    """Scale 2^(floor(log2 amax) - 8), stored with bias 127; the block max may sit anywhere in
    its 32 elements."""
    rng = np.random.default_rng(j + 100 + 1000 * pos)
    for f in (1.0, 1.4, 1.999):
        blk = rng.uniform(-1.0, 1.0, 32) * 2.0 ** j
        blk[pos] = -f * 2.0 ** j
        codes, scales = oracle.mx_quantize(blk)
        assert scales[0] == 127 + j - 8
        assert codes[pos] == oracle.e4m3_encode(-f * 256.0)


def test_zero_block():
    codes, scales = oracle.mx_quantize(np.zeros(64))
    assert scales.tolist() == [0, 0] and not codes.any()


def test_blocks_are_independent():
    v = np.concatenate([np.full(32, 3.0e-3), np.full(32, 5.0e4)])
    v[5], v[40] = 1.7e-3, -2.2e4
    codes, scales = oracle.mx_quantize(v)
    c0, s0 = oracle.mx_quantize(v[:32])
    c1, s1 = oracle.mx_quantize(v[32:])
    np.testing.assert_array_equal(codes, np.concatenate([c0, c1]))
    np.testing.assert_array_equal(scales, np.concatenate([s0, s1]))
    assert scales[0] == 127 + math.floor(math.log2(3.0e-3)) - 8
    assert scales[1] == 127 + math.floor(math.log2(5.0e4)) - 8


def test_small_element_under_a_large_maximum():
    """448 fixes s = 0, so 5 * 2^-11 (below E4M3's smallest normal) rounds on the subnormal grid
    of spacing 2^-9: 1.25 steps -> 1 step."""
    v = np.zeros(32)
    v[0], v[1] = 448.0, 5 * 2.0 ** -11
    codes, scales = oracle.mx_quantize(v)
    assert scales[0] == 127 and codes[0] == 0x7E and codes[1] == 0x01


def test_grid_data_round_trips_exactly():
    """Blocks built from E4M3 codes and a scale, with one element in E4M3's top binade (so the
    scale rule picks that scale back), are quantised to exactly those codes."""
    rng = np.random.default_rng(3)
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    for _ in range(200):
        codes = rng.choice(finite, 32).astype(np.uint8)
        codes[rng.integers(32)] = rng.integers(0x78, 0x7F) | (0x80 * rng.integers(2))
        s = int(rng.integers(-100, 100))
        v = oracle.mx_values(codes, np.array([s + 127]))
        c2, s2 = oracle.mx_quantize(v)
        assert s2[0] == s + 127
        np.testing.assert_array_equal(oracle.mx_values(c2, s2), v)


def test_rounding_error_bound():
    """Elements at or above E4M3's smallest normal (2^-6 X) err by at most half a step of a
    3-bit mantissa, 2^-4 relative; elements below it by at most half the subnormal step,
    2^-10 X."""
    rng = np.random.default_rng(11)
    v = rng.standard_normal(32 * 400) * np.exp2(rng.integers(-30, 30, 32 * 400) / 4.0)
    codes, scales = oracle.mx_quantize(v)
    q = oracle.mx_values(codes, scales)
    X = np.repeat(np.exp2(scales.astype(np.float64) - 127), 32)
    a = np.abs(v) / X
    assert a.max() <= 512.0
    normal = (a >= 2.0 ** -6) & (a <= 448.0)
    assert np.all(np.abs(q - v)[normal] <= 2.0 ** -4 * np.abs(v)[normal] * (1 + 1e-12))
    sub = a < 2.0 ** -6
    assert np.all(np.abs(q - v)[sub] <= 2.0 ** -10 * X[sub] * (1 + 1e-12))
    big = a > 448.0
    assert np.all(np.abs(q[big]) == 448.0 * X[big])


def test_bf16_row_quantiser_matches_the_vector_one():
    g = torch.Generator().manual_seed(5)
    m = (torch.randn(9, 96, generator=g) * torch.exp2(torch.randint(-6, 6, (9, 1), generator=g).float())
         ).to(torch.bfloat16)
    codes, scales = oracle.mx_quantize_bf16_rows(m)
    for r in range(9):
        c, s = oracle.mx_quantize(m[r].double().numpy())
        np.testing.assert_array_equal(codes[r], c)
        np.testing.assert_array_equal(scales[r], s)


# ----------------------------------------------------------------------------------------
# the layer with MXFP8 experts
# ----------------------------------------------------------------------------------------

def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        fx = json.load(f)
    inp = {k: _bf16(fx[k]) for k in ("x", "W_router", "W_up", "W_gate", "W_down")}
    for k in ("Ws_up", "Ws_gate", "Ws_down"):
        inp[k] = _bf16(fx[k]) if k in fx else None
    inp["bias"] = None
    return fx, inp


def test_hand_worked_mx_layer():
    fx, inp = _load("mx_hand_worked_layer.json")
    res = oracle.forward(inp, fx["top_k"], block_m=2, mxfp8=True)
    np.testing.assert_array_equal(res["topk_ids"], [[0]])
    np.testing.assert_allclose(res["out"], np.array(fx["expect"]["out"], dtype=np.float64),
                               rtol=0, atol=1e-15)


def _rand_inputs(T=12, H=64, D=64, E=4, Ds=32, seed=0):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s, sc=1.0: (sc * torch.randn(*s, generator=g)).to(torch.bfloat16)
    inp = {"x": r(T, H), "W_router": r(E, H, sc=0.2), "bias": None,
           "W_up": r(E, D, H, sc=0.15), "W_gate": r(E, D, H, sc=0.15), "W_down": r(E, H, D, sc=0.15)}
    if Ds:
        inp.update(Ws_up=r(Ds, H, sc=0.15), Ws_gate=r(Ds, H, sc=0.15), Ws_down=r(H, Ds, sc=0.15))
    else:
        inp.update(Ws_up=None, Ws_gate=None, Ws_down=None)
    return inp


def test_power_of_two_scalings_commute_with_quantisation():
    """Scaling W_down by 2 doubles every output; scaling W_gate by 4 scales h, and so its
    MX quantisation, by 4, and the output with it; both exactly."""
    inp = _rand_inputs()
    base = oracle.forward(inp, 2, block_m=16, mxfp8=True)["out"]
    s2 = dict(inp, W_down=(inp["W_down"].float() * 2).to(torch.bfloat16),
              Ws_down=(inp["Ws_down"].float() * 2).to(torch.bfloat16))
    np.testing.assert_array_equal(oracle.forward(s2, 2, block_m=16, mxfp8=True)["out"], 2 * base)
    s4 = dict(inp, W_gate=(inp["W_gate"].float() * 4).to(torch.bfloat16),
              Ws_gate=(inp["Ws_gate"].float() * 4).to(torch.bfloat16))
    np.testing.assert_array_equal(oracle.forward(s4, 2, block_m=16, mxfp8=True)["out"], 4 * base)


def test_grid_weights_and_inputs_leave_only_h_rounding():
    """With x and every weight already on the MX grid, the only difference from the exact
    layer is h's rounding, which is at most 2^-4 relative per element of h."""
    inp = _rand_inputs(Ds=0, seed=4)

    def on_grid(t):
        c, s = oracle.mx_quantize_bf16_rows(t.reshape(-1, t.shape[-1]))
        v = oracle.mx_values(c.ravel(), s.ravel()).reshape(t.shape)
        return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16)

    g = dict(inp, x=on_grid(inp["x"]), W_up=on_grid(inp["W_up"]), W_gate=on_grid(inp["W_gate"]),
             W_down=on_grid(inp["W_down"]))
    for k in ("x", "W_up", "W_gate", "W_down"):
        assert torch.equal(on_grid(g[k]), g[k])
    mx = oracle.forward(g, 2, block_m=16, mxfp8=True)
    ex = oracle.forward(g, 2, block_m=16)
    # bound: sum over slots of w * sum_d |W_down[h, d]| * 2^-4 |h_d|, with |h_d| from the
    # exact layer's own h (recomputed here in float64 from the grid values)
    x = g["x"].double().numpy()
    bound = np.zeros_like(ex["out"])
    for t in range(x.shape[0]):
        for j in range(2):
            e = mx["topk_ids"][t, j]
            u = g["W_up"][e].double().numpy() @ x[t]
            gg = g["W_gate"][e].double().numpy() @ x[t]
            h = u / (1 + np.exp(-u)) * gg
            bound[t] += mx["topk_w"][t, j] * (np.abs(g["W_down"][e].double().numpy()) @ (np.abs(h) * 2.0 ** -4 * 1.0001 + 1e-30))
    assert np.all(np.abs(mx["out"] - ex["out"]) <= bound)
    assert np.any(mx["out"] != ex["out"])


def _mx_rows(t):
    """Values of the MX quantisation of each row of a bf16 matrix, float64."""
    m = t.reshape(-1, t.shape[-1])
    c, s = oracle.mx_quantize_bf16_rows(m)
    return oracle.mx_values(c.ravel(), s.ravel()).reshape(m.shape)


def test_mx_expert_h_is_swiglu_of_the_quantised_operands():
    """The MXFP8 layer's GEMM1 stage against numpy on the quantiser's own values: u = Wq_up xq,
    g = Wq_gate xq, h = fp32(SiLU(u) g), with the |Wq xq| sums; the shared expert's rows hold Ds
    entries; and from h, the layer's remaining steps (h quantised, Wq_down, weighted sum in slot
    order) written out with numpy give the layer's output."""
    inp = _rand_inputs(T=10, H=64, D=64, E=4, Ds=32, seed=9)
    E = 4
    rng = np.random.default_rng(2)
    tokens = rng.integers(0, 10, size=24)
    experts = rng.integers(0, E + 1, size=24).astype(np.int32)
    h, u, g, au, ag = oracle.expert_h(inp["x"], inp, tokens, experts, with_parts=True, mxfp8=True)
    xq = _mx_rows(inp["x"])
    for i, (t, e) in enumerate(zip(tokens, experts)):
        wu = _mx_rows(inp["Ws_up"] if e == E else inp["W_up"][e])
        wg = _mx_rows(inp["Ws_gate"] if e == E else inp["W_gate"][e])
        n = wu.shape[0]
        ur, gr = wu @ xq[t], wg @ xq[t]
        np.testing.assert_allclose(u[i, :n], ur, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(g[i, :n], gr, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(au[i, :n], np.abs(wu) @ np.abs(xq[t]), rtol=1e-12)
        np.testing.assert_allclose(ag[i, :n], np.abs(wg) @ np.abs(xq[t]), rtol=1e-12)
        np.testing.assert_allclose(h[i, :n], (ur / (1 + np.exp(-ur)) * gr).astype(np.float32), rtol=2e-7, atol=1e-30)
    res = oracle.forward(inp, 2, block_m=16, mxfp8=True)
    T = inp["x"].shape[0]
    tk = np.repeat(np.arange(T), 3)
    ex = np.concatenate([np.full((T, 1), E), res["topk_ids"]], axis=1).reshape(-1).astype(np.int32)
    hh = oracle.expert_h(inp["x"], inp, tk, ex, mxfp8=True)
    out = np.zeros((T, inp["x"].shape[1]))
    for i, (t, e) in enumerate(zip(tk, ex)):
        wd = _mx_rows(inp["Ws_down"] if e == E else inp["W_down"][e])
        c, s = oracle.mx_quantize(hh[i, :wd.shape[1]])
        y = wd @ oracle.mx_values(c, s)
        j = i % 3
        out[t] += y if j == 0 else res["topk_w"][t, j - 1] * y
    np.testing.assert_allclose(out, res["out"], rtol=1e-12, atol=1e-13)
