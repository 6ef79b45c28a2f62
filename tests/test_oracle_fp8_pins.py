"""Pins of the oracle's FP8 E4M3 routed-expert path (dequantize on load, 128x128 block
scales: miles Step-5-Preview page, section 1 "FP8 checkpoint").

Each pin ties the oracle to something outside it: torch's float8_e4m3fn conversion (a
library routine), closed-form code values of the E4M3 format, a numpy restatement of
the block-scale indexing, and the BF16 oracle on weights that both paths represent
exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_layer_biased_b200.inputs import LayerShape, bf16_bits, draw, draw_fp8

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _torch_e4m3(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def test_e4m3_decode_matches_torch_on_every_code():
    v = oracle.e4m3_values()
    t = _torch_e4m3(np.arange(256)).astype(np.float64)
    assert np.array_equal(np.isnan(v), np.isnan(t))
    assert np.array_equal(v[~np.isnan(v)], t[~np.isnan(t)])


def test_e4m3_closed_form_codes():
    v = oracle.e4m3_values()
    assert v[0x00] == 0.0 and np.signbit(v[0x80])
    assert v[0x38] == 1.0 and v[0xB8] == -1.0  # exponent field 7 = bias, mantissa 0
    assert v[0x01] == 2.0**-9  # smallest subnormal: 1/8 * 2^-6
    assert v[0x08] == 2.0**-6  # smallest normal
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0  # largest finite: 1.75 * 2^8
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])  # the only NaN codes, no infinities
    assert np.isfinite(v[[c for c in range(256) if c not in (0x7F, 0xFF)]]).all()


def test_dequant_block_indexing_on_ragged_matrix():
    rng = np.random.default_rng(5)
    rows, cols = 300, 200  # blocks 3 x 2 with partial last row and column blocks
    q = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
    q[q == 0x7F] = 0x7E
    q[q == 0xFF] = 0xFE
    s = rng.uniform(0.25, 4.0, size=(3, 2)).astype(np.float32)
    got = oracle.dequant_block128(q, s)
    want = _torch_e4m3(q) * np.repeat(np.repeat(s, 128, 0), 128, 1)[:rows, :cols]
    assert got.dtype == np.float32
    np.testing.assert_array_equal(got, want.astype(np.float32))


SMALL = LayerShape("fp8_small", T=24, H=256, E=4, k=2, I=256, Is=128, limit_routed=0.25,
                   limit_shared=0.125, seed=41, weight_std=0.03)


def test_f32_weight_experts_equal_bf16_oracle_on_bf16_weights():
    """Same weights (bf16 values held in fp32): the fp32-weight expert pass and the BF16
    given-routing oracle are the same sums in the same order."""
    sh = SMALL
    inp = draw(sh)
    x = bf16_bits(inp["x"])
    r = oracle.router(x, bf16_bits(inp["Wr"]), inp["bias"].numpy(), sh.k)
    w32 = r["w"].astype(np.float32)
    gu, d = bf16_bits(inp["W_gate_up"]), bf16_bits(inp["W_down"])
    ref = oracle.forward_given_routing(x, r["idx"], w32, {e: (gu[e], d[e]) for e in range(sh.E)},
                                       bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), E=sh.E,
                                       limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    f32 = {e: (inp["W_gate_up"][e].float().numpy(), inp["W_down"][e].float().numpy()) for e in range(sh.E)}
    got = oracle.experts_f32w(x, r["idx"], w32.astype(np.float64), f32, bf16_bits(inp["Wsh_gate_up"]),
                              bf16_bits(inp["Wsh_down"]), E=sh.E, limit_routed=sh.limit_routed,
                              limit_shared=sh.limit_shared)
    np.testing.assert_array_equal(got, ref)


def test_fp8_forward_equals_bf16_forward_with_power_of_two_block_scales():
    """With power-of-two block scales every dequantized weight (4 significant bits times
    2^j) is exact in bf16, so the FP8 layer must equal the BF16 oracle on those bf16
    weights: pins the gate/up/down block indexing and the expert plumbing."""
    sh = SMALL
    inp = draw_fp8(sh)
    rng = np.random.default_rng(7)
    sgu = np.ldexp(1.0, rng.integers(-14, -10, size=inp["W_gate_up_s"].shape)).astype(np.float32)
    sd = np.ldexp(1.0, rng.integers(-14, -10, size=inp["W_down_s"].shape)).astype(np.float32)
    assert len(np.unique(sgu)) > 1 and len(np.unique(sd)) > 1
    qgu, qd = inp["W_gate_up_q"].numpy(), inp["W_down_q"].numpy()
    x, Wr, bias = bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy()
    shg, shd = bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"])
    got = oracle.forward_fp8_tokens(x, Wr, bias, qgu, sgu, qd, sd, shg, shd, k=sh.k,
                                    limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)

    def bf16_of(q, s):
        w = _torch_e4m3(q) * np.repeat(np.repeat(s, 128, 0), 128, 1)[: q.shape[0], : q.shape[1]]
        b = torch.from_numpy(w).to(torch.bfloat16)
        assert torch.equal(b.float(), torch.from_numpy(w))  # exact in bf16
        return b.view(torch.int16).numpy().view(np.uint16)

    experts = {e: (bf16_of(qgu[e], sgu[e]), bf16_of(qd[e], sd[e])) for e in range(sh.E)}
    ref = oracle.forward_tokens(x, Wr, bias, experts, shg, shd, k=sh.k, limit_routed=sh.limit_routed,
                                limit_shared=sh.limit_shared)
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    np.testing.assert_array_equal(got["y"], ref["y"])


def test_fp8_draw_shares_router_inputs_and_spreads_codes():
    sh = SMALL
    a, b = draw_fp8(sh), draw(sh)
    for key in ("x", "Wr", "bias"):
        assert torch.equal(a[key], b[key])
    v = _torch_e4m3(a["W_gate_up_q"].numpy())
    assert np.isfinite(v).all() and np.abs(v).max() <= 448.0
    assert 50.0 < v.std() < 80.0
    assert a["W_gate_up_s"].shape == (sh.E, 2 * sh.I // 128, sh.H // 128)
    assert a["W_down_s"].shape == (sh.E, sh.H // 128, sh.I // 128)
