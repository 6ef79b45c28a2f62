"""GPU parity of the FP8 E4M3 routed-expert path (moe_forward_fp8) against the oracle.

The oracle dequantizes the selected experts (e4m3 code * 128x128 block scale, fp32) and
runs the layer in double; the GPU streams the codes and multiplies by bf16(e4m3 *
scale) on the tensor cores. The extra bf16 rounding of each dequantized weight
(relative <= 2^-9, independent across weights) adds about 2^-9 / sqrt(3) ~ 1.1e-3
relative error to a dot product whose terms have random signs, inside the layer's
1e-2 relative-Frobenius / 3e-2 max-abs bar, which the tests keep.

Decode-sized calls with H a multiple of 256 and I, Is multiples of 128 run the routed experts
on the FP8 tensor cores instead (E4M3 codes straight into the MMA, each block scale and each
token row's largest |x| applied to the token operand, which is split into two E4M3 parts
carrying about 8 significant bits: the precision of the bf16 operands above).
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import check_output, check_routing, rel_fro
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import WORKLOADS, LayerShape, bf16_bits, draw_fp8, token_sample
from sparse_moe_layer_biased_b200.layer import MoeLayer

pytestmark = pytest.mark.gpu

SHAPES = {
    # decode-sized (<= 16 tokens per expert on average): 32-row chunks
    "tiny": WORKLOADS["tiny"],
    "decode": LayerShape("fp8_decode", T=24, H=512, E=40, k=8, I=256, Is=128, limit_routed=0.25, seed=51,
                         weight_std=0.03),
    # decode stages span 128 K elements: the shared expert's down GEMM (K = Is = 192) ends
    # in a half-empty stage that TMA fills with zeros for both operands
    "decode_is192": LayerShape("fp8_decode_is192", T=24, H=512, E=40, k=8, I=256, Is=192, limit_shared=0.25,
                               seed=55, weight_std=0.03),
    # decode-sized with H a multiple of 256 and I, Is of 128: the FP8 tensor-core kernels
    # (E4M3 weights straight into the MMA, block scales on the token operand); 6 K blocks of
    # gate/up, 3 down tiles of 256 rows, 2 shared feature blocks, chunks of 16 and 32 rows
    "decode_h768": LayerShape("fp8_decode_h768", T=40, H=768, E=24, k=6, I=256, Is=256, limit_routed=0.25,
                              seed=58, weight_std=0.03),
    # FP8 tensor-core edge cases: a single token (every chunk one row, 15 padding rows of the
    # 16-row operand), and every expert selected by every token (k = E)
    "one_token": LayerShape("fp8_one_token", T=1, H=256, E=8, k=2, I=128, Is=128, seed=61, weight_std=0.03),
    "all_experts": LayerShape("fp8_all_experts", T=5, H=512, E=8, k=8, I=256, Is=128, limit_routed=0.25,
                              seed=62, weight_std=0.03),
    # prefill-sized: 128-row chunks, several K blocks, ragged chunk tails, Is not a multiple of 128
    "prefill": LayerShape("fp8_prefill", T=300, H=512, E=12, k=4, I=256, Is=192, limit_routed=0.25,
                          limit_shared=0.125, seed=52, weight_std=0.03),
    # prefill-sized, wider: 6 K blocks of gate/up, 6 down row blocks, 4 shared-expert
    # gate/up feature blocks, ragged chunk tails
    "prefill_h768": LayerShape("fp8_prefill_h768", T=333, H=768, E=10, k=4, I=384, Is=256, limit_routed=0.25,
                               limit_shared=0.125, seed=56, weight_std=0.03),
    # prefill-sized with I, Is multiples of 128 and H of 512: the BF16 shared expert runs on
    # the CTA-pair kernels (its own tile tables), the routed experts on the FP8 kernels
    "prefill_pair": LayerShape("fp8_prefill_pair", T=300, H=512, E=12, k=4, I=256, Is=256, limit_routed=0.25,
                               limit_shared=0.125, seed=57, weight_std=0.03),
    "ragged": LayerShape("fp8_ragged", T=333, H=384, E=40, k=6, I=128, Is=320, limit_routed=0.0,
                         limit_shared=0.0, seed=53, weight_std=0.03),
    # pre-activations of std ~1 against routed limit 0.5: the up clamp binds on ~60% and
    # the silu cap on ~20% of routed units (outputs stay at the workloads' scale, where
    # the absolute bar applies)
    "clip": LayerShape("fp8_clip", T=200, H=256, E=8, k=2, I=384, Is=128, limit_routed=0.5, limit_shared=0.25,
                       seed=54, weight_std=0.06),
}


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    _abi.lib()
    yield
    _abi.moe_check_device()


def _oracle(sh, inp, rows=None):
    """Oracle layer output (fp64) for the listed rows of a host-resident FP8 draw."""
    x = inp["x"] if rows is None else inp["x"][rows]
    return oracle.forward_fp8_tokens(
        bf16_bits(x), bf16_bits(inp["Wr"]), inp["bias"].numpy(), inp["W_gate_up_q"].numpy(),
        inp["W_gate_up_s"].numpy(), inp["W_down_q"].numpy(), inp["W_down_s"].numpy(),
        bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), k=sh.k, scale=sh.scale,
        norm=sh.norm_expert_weight, limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)


def _forward(sh, inp_dev, det=False):
    layer = MoeLayer(sh, inp_dev, deterministic=det)
    assert layer.fp8
    y, idx, w = layer.forward(inp_dev["x"], routing=True)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    return y.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("name", list(SHAPES))
def test_fp8_forward_small(name, det):
    sh = SHAPES[name]
    inp = draw_fp8(sh)
    y, idx, w = _forward(sh, {k: v.cuda() for k, v in inp.items()}, det)
    ref = _oracle(sh, inp)
    keep = check_routing(idx, w, ref, sh.E, sh.k)
    rf, ma = check_output(y[keep], ref["y"][keep], name)
    print(f"{name} det={det}: rel_fro {rf:.2e} max_abs {ma:.2e}")


def test_fp8_deterministic_matches_atomic():
    sh = SHAPES["prefill"]
    inp = {k: v.cuda() for k, v in draw_fp8(sh).items()}
    ya, _, _ = _forward(sh, inp, det=False)
    yd, _, _ = _forward(sh, inp, det=True)
    yd2, _, _ = _forward(sh, inp, det=True)
    np.testing.assert_array_equal(yd, yd2)
    assert rel_fro(ya, yd) < 1e-6


def test_fp8_scales_are_applied_per_block():
    """Doubling every scale of one expert's down projection doubles that expert's
    contribution: y(2s) - y(s) equals the difference the oracle predicts."""
    sh = SHAPES["prefill"]
    inp = draw_fp8(sh)
    dev = {k: v.cuda() for k, v in inp.items()}
    y1, idx, _ = _forward(sh, dev, det=True)
    e = int(np.bincount(idx.ravel(), minlength=sh.E).argmax())
    inp2 = dict(inp)
    s2 = inp["W_down_s"].clone()
    s2[e] *= 2.0
    inp2["W_down_s"] = s2
    dev["W_down_s"] = s2.cuda()
    y2, _, _ = _forward(sh, dev, det=True)
    r1, r2 = _oracle(sh, inp), _oracle(sh, inp2)
    check_output(y2 - y1, r2["y"] - r1["y"], "scale delta")


@pytest.fixture(scope="module", params=["step35_decode", "step35_prefill"])
def full(request):
    sh = WORKLOADS[request.param]
    inp = draw_fp8(sh, device="cuda")
    y, idx, w = _forward(sh, inp)
    yield {"shape": sh, "inp": inp, "y": y, "idx": idx, "w": w}
    del inp
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_fp8_full_size_output_sampled(full):
    """Full-size shapes in the benchmark's launch configuration: routing of the sampled
    tokens and their outputs against the oracle (only their experts are dequantized)."""
    sh = full["shape"]
    rows = token_sample(sh.T, 4, sh.seed).numpy()
    inp = full["inp"]
    x_rows = inp["x"][torch.from_numpy(rows).cuda()]
    r = oracle.router(bf16_bits(x_rows), bf16_bits(inp["Wr"]), inp["bias"].cpu().numpy(), sh.k)
    ids = sorted(set(int(e) for e in r["idx"].ravel()))
    experts = {e: (oracle.dequant_block128(inp["W_gate_up_q"][e].cpu().numpy(), inp["W_gate_up_s"][e].cpu().numpy()),
                   oracle.dequant_block128(inp["W_down_q"][e].cpu().numpy(), inp["W_down_s"][e].cpu().numpy()))
               for e in ids}
    y_ref = oracle.experts_f32w(bf16_bits(x_rows), r["idx"], r["w"], experts, bf16_bits(inp["Wsh_gate_up"]),
                                bf16_bits(inp["Wsh_down"]), E=sh.E, limit_routed=sh.limit_routed,
                                limit_shared=sh.limit_shared)
    keep = r["margin"] >= 1e-6
    np.testing.assert_array_equal(np.sort(full["idx"][rows][keep], 1), np.sort(r["idx"][keep], 1))
    rf, ma = check_output(full["y"][rows][keep], y_ref[keep], sh.name)
    print(f"{sh.name} fp8 sampled: rel_fro {rf:.2e} max_abs {ma:.2e}")


def test_fp8_decode_row_and_block_scaling():
    """FP8 tensor-core decode path: the token operand is scaled per row by its largest |x|
    and per weight block row by its largest block scale. Rows of very different magnitude
    (x 8, x 2^-6: the layer's relative bar, row by row; all zero: output exactly 0) and block
    scales spread over a factor 2^8 within each block row (the layer bar on the other rows)."""
    sh = SHAPES["decode_h768"].replace(limit_routed=0.0)
    inp = draw_fp8(sh)
    x = inp["x"].float()
    x[0] *= 8.0
    x[1] *= 2.0 ** -6
    x[2] = 0.0
    inp["x"] = x.to(torch.bfloat16)
    gen = torch.Generator().manual_seed(59)
    for key in ("W_gate_up_s", "W_down_s"):
        # factors 2^-4 .. 2^4 along each block row (K blocks), renormalised so the row's
        # mean square is kept: the outputs stay at the workload's scale, where the absolute
        # bar applies
        spread = torch.exp2(torch.randint(-4, 5, inp[key].shape, generator=gen).float())
        spread = spread / spread.square().mean(-1, keepdim=True).sqrt()
        inp[key] = inp[key] * spread
    y, idx, w = _forward(sh, {k: v.cuda() for k, v in inp.items()})
    ref = _oracle(sh, inp)
    keep = check_routing(idx, w, ref, sh.E, sh.k)
    assert np.abs(y[2]).max() == 0.0
    for r in (0, 1):
        if not keep[r]:
            continue  # a near tie: the routing check above covers it
        rf = rel_fro(y[r], ref["y"][r])
        print(f"row {r}: rel_fro {rf:.2e}")
        assert rf <= 1e-2
    rest = keep.copy()
    rest[:3] = False
    rf, ma = check_output(y[rest], ref["y"][rest], "scaled rows")
    print(f"decode_h768 scaled: rel_fro {rf:.2e} max_abs {ma:.2e}")


def test_fp8_decode_scales_are_applied_per_block():
    """FP8 tensor-core decode path: doubling every down scale of the busiest expert doubles
    its contribution (the difference matches the oracle's)."""
    sh = SHAPES["decode_h768"]
    inp = draw_fp8(sh)
    dev = {k: v.cuda() for k, v in inp.items()}
    y1, idx, _ = _forward(sh, dev, det=True)
    e = int(np.bincount(idx.ravel(), minlength=sh.E).argmax())
    inp2 = dict(inp)
    s2 = inp["W_down_s"].clone()
    s2[e] *= 2.0
    inp2["W_down_s"] = s2
    dev["W_down_s"] = s2.cuda()
    y2, _, _ = _forward(sh, dev, det=True)
    r1, r2 = _oracle(sh, inp), _oracle(sh, inp2)
    check_output(y2 - y1, r2["y"] - r1["y"], "decode scale delta")


def test_fp8_decode_extreme_codes():
    """FP8 tensor-core decode path on codes at the ends of the E4M3 range: the largest
    finite magnitudes (448, codes 0x7e / 0xfe), every subnormal code (0x01..0x07 and their
    negatives) and zeros, mixed into the drawn weights, against the oracle's exact decode
    (routed clip off, so the routed experts carry most of the output)."""
    sh = SHAPES["decode_h768"].replace(limit_routed=0.0)
    inp = draw_fp8(sh)
    gen = torch.Generator().manual_seed(60)
    special = torch.tensor([0x7E, 0xFE, 0x00, 0x80] + list(range(0x01, 0x08)) + list(range(0x81, 0x88)),
                           dtype=torch.uint8)
    for key in ("W_gate_up_q", "W_down_q"):
        q = inp[key].clone()
        mask = torch.rand(q.shape, generator=gen) < 0.05
        pick = torch.randint(0, special.numel(), q.shape, generator=gen)
        q[mask] = special[pick[mask]]
        inp[key] = q
    y, idx, w = _forward(sh, {k: v.cuda() for k, v in inp.items()})
    ref = _oracle(sh, inp)
    keep = check_routing(idx, w, ref, sh.E, sh.k)
    rf, ma = check_output(y[keep], ref["y"][keep], "extreme codes")
    print(f"decode_h768 extreme codes: rel_fro {rf:.2e} max_abs {ma:.2e}")
