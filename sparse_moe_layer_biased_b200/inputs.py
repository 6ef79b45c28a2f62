"""Seeded synthetic inputs for the biased-sigmoid MoE FFN layer.

This module only draws tensors: it holds none of the layer's arithmetic, and it
imports nothing else from this package. The CPU oracle (tests) and the CUDA
path both receive the tensors it returns.

Workloads follow the Step-3.5-Flash / Step-5-Preview MoE layer shapes:
- "MAX 中 Step-3.5-Flash 架构解析", section "Step3p5Config配置项全解": 288 routed
  experts, top-8, expert and shared-expert intermediate 1280, routing scale 3.0,
  normalised expert weights, per-layer SwiGLU limits (0 = no clip).
- NeMo AutoModel Step-5-Preview page, "Model Architecture" table: hidden 4096,
  352 routed experts, top-8, intermediate 1536 for routed and shared experts.

Recipe (fixed draw order, one torch.Generator seeded per workload):
  x ~ N(0, 1), Wr ~ N(0, 0.02^2), W_gate_up ~ N(0, 0.02^2), W_down ~ N(0, 0.02^2),
  Wsh_gate_up ~ N(0, 0.02^2), Wsh_down ~ N(0, 0.02^2): drawn in fp32, rounded to
  bf16 (round-to-nearest-even); router bias ~ U(-0.1, 0.1) in fp32.
  Draw order: x, Wr, bias, W_gate_up (expert by expert), W_down (expert by
  expert), Wsh_gate_up, Wsh_down.
  The skewed workload replaces the uniform bias by a Zipf-shaped log-rank bias
  over a random expert permutation: bias[perm[r]] = -gamma * s * ln(r + 1),
  s = 1.1, with gamma fixed so that the hottest 8 experts take about 30% of the
  assignments (gamma comes from oracle/calibrate_zipf.py).

Layouts (row-major, K innermost, PyTorch [out, in] convention):
  x [T, H] bf16; Wr [E, H] bf16; bias [E] fp32;
  W_gate_up [E, 2I, H] bf16 (rows [0, I) gate, rows [I, 2I) up);
  W_down [E, H, I] bf16; Wsh_gate_up [2Is, H] bf16; Wsh_down [H, Is] bf16.

FP8 variant (draw_fp8): the routed experts as FP8 E4M3 codes with one fp32 scale per
128x128 block, the format of the Step-5-Preview checkpoint (miles Step-5-Preview page,
section 1); x, Wr, bias and the BF16 shared expert as above.
"""
from __future__ import annotations

import dataclasses

import torch

ZIPF_S = 1.1
# Written by oracle/calibrate_zipf.py (CPU oracle router, 4096 tokens drawn like
# the skewed workload): hottest-8 share of assignments = 0.30 at this gamma.
ZIPF_GAMMA = 0.081537
# Spread of the drawn FP8 E4M3 codes (draw_fp8): most of the format's range below 448.
FP8_CODE_STD = 64.0


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """One MoE layer workload. Field names follow Step3p5Config keys."""

    name: str
    T: int  # tokens
    H: int  # hidden size
    E: int  # moe_num_experts
    k: int  # moe_top_k
    I: int  # moe_intermediate_size
    Is: int  # share_expert_dim
    scale: float = 3.0  # moe_router_scaling_factor
    norm_expert_weight: bool = True
    limit_routed: float = 0.0  # swiglu_limits[layer]; 0 = no clip
    limit_shared: float = 0.0  # swiglu_limits_shared[layer]; 0 = no clip
    seed: int = 0
    bias_kind: str = "uniform"  # "uniform" or "zipf"
    weight_std: float = 0.02
    x_std: float = 1.0

    def replace(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)

    @property
    def flops_per_token(self) -> float:
        """Algorithmic FLOPs per token: router GEMV + k routed + 1 shared SwiGLU MLP."""
        return 2.0 * self.H * self.E + 6.0 * self.H * self.I * self.k + 6.0 * self.H * self.Is


WORKLOADS = {
    "tiny": LayerShape("tiny", T=64, H=256, E=16, k=4, I=128, Is=128,
                       limit_routed=7.0, limit_shared=0.0, seed=0),
    "step35_prefill": LayerShape("step35_prefill", T=4096, H=4096, E=288, k=8, I=1280, Is=1280,
                                 limit_routed=7.0, limit_shared=0.0, seed=1),
    "step35_decode": LayerShape("step35_decode", T=64, H=4096, E=288, k=8, I=1280, Is=1280,
                                limit_routed=7.0, limit_shared=0.0, seed=2),
    "step5_prefill": LayerShape("step5_prefill", T=8192, H=4096, E=352, k=8, I=1536, Is=1536,
                                limit_routed=0.0, limit_shared=0.0, seed=3),
    "step5_skewed": LayerShape("step5_skewed", T=16384, H=4096, E=352, k=8, I=1536, Is=1536,
                               limit_routed=7.0, limit_shared=0.0, seed=4, bias_kind="zipf"),
}


def zipf_bias(E: int, seed: int, gamma: float, s: float = ZIPF_S) -> torch.Tensor:
    """Log-rank bias over a seeded random expert permutation (CPU generator)."""
    g = torch.Generator().manual_seed(1_000_003 + seed)
    perm = torch.randperm(E, generator=g)
    bias = torch.empty(E, dtype=torch.float32)
    ranks = torch.arange(E, dtype=torch.float64)
    bias[perm] = (-gamma * s * torch.log1p(ranks)).to(torch.float32)
    return bias


def _normal_bf16(shape, std, gen, device):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def draw(shape: LayerShape, device="cpu", gamma: float | None = None) -> dict:
    """Draw every input of one layer call on `device` (same recipe on CPU and CUDA).

    The draw is deterministic for a given (shape, device type). Large weights are
    drawn one expert at a time so the fp32 temporaries stay small.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(shape.seed)
    T, H, E, I, Is = shape.T, shape.H, shape.E, shape.I, shape.Is
    out = {}
    out["x"] = _normal_bf16((T, H), shape.x_std, gen, dev)
    out["Wr"] = _normal_bf16((E, H), shape.weight_std, gen, dev)
    bias = torch.rand((E,), generator=gen, device=dev, dtype=torch.float32).mul_(0.2).sub_(0.1)
    wgu = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, device=dev)
    for e in range(E):
        wgu[e] = _normal_bf16((2 * I, H), shape.weight_std, gen, dev)
    wd = torch.empty((E, H, I), dtype=torch.bfloat16, device=dev)
    for e in range(E):
        wd[e] = _normal_bf16((H, I), shape.weight_std, gen, dev)
    out["W_gate_up"] = wgu
    out["W_down"] = wd
    out["Wsh_gate_up"] = _normal_bf16((2 * Is, H), shape.weight_std, gen, dev)
    out["Wsh_down"] = _normal_bf16((H, Is), shape.weight_std, gen, dev)
    if shape.bias_kind == "zipf":
        g = ZIPF_GAMMA if gamma is None else gamma
        bias = zipf_bias(E, shape.seed, g).to(dev)
    out["bias"] = bias
    return out


def _e4m3_codes(shape, gen, device):
    """FP8 E4M3 codes (uint8) of N(0, 64^2) draws, clamped to the format's +-448 range and
    rounded to nearest even by torch's float8_e4m3fn cast."""
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32).mul_(FP8_CODE_STD)
    return t.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def draw_fp8(shape: LayerShape, device="cpu", gamma: float | None = None) -> dict:
    """Inputs of one layer call with FP8 E4M3 routed experts (128x128 block scales).

    x, Wr, bias and the BF16 shared expert are drawn exactly as draw() draws them; the
    routed experts are drawn as E4M3 codes ~ N(0, 64^2) (W_gate_up_q [E, 2I, H],
    W_down_q [E, H, I], uint8) with one fp32 scale per 128x128 block,
    scale ~ (weight_std / 64) * U(0.5, 1.5) (W_gate_up_s [E, ceil(2I/128), ceil(H/128)],
    W_down_s [E, ceil(H/128), ceil(I/128)]), so a dequantized weight has about the
    BF16 draw's spread. Draw order: x, Wr, bias, W_gate_up_q (expert by expert),
    W_down_q (expert by expert), Wsh_gate_up, Wsh_down, W_gate_up_s, W_down_s.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(shape.seed)
    T, H, E, I, Is = shape.T, shape.H, shape.E, shape.I, shape.Is
    out = {}
    out["x"] = _normal_bf16((T, H), shape.x_std, gen, dev)
    out["Wr"] = _normal_bf16((E, H), shape.weight_std, gen, dev)
    bias = torch.rand((E,), generator=gen, device=dev, dtype=torch.float32).mul_(0.2).sub_(0.1)
    qgu = torch.empty((E, 2 * I, H), dtype=torch.uint8, device=dev)
    for e in range(E):
        qgu[e] = _e4m3_codes((2 * I, H), gen, dev)
    qd = torch.empty((E, H, I), dtype=torch.uint8, device=dev)
    for e in range(E):
        qd[e] = _e4m3_codes((H, I), gen, dev)
    out["W_gate_up_q"] = qgu
    out["W_down_q"] = qd
    out["Wsh_gate_up"] = _normal_bf16((2 * Is, H), shape.weight_std, gen, dev)
    out["Wsh_down"] = _normal_bf16((H, Is), shape.weight_std, gen, dev)
    blk = lambda n: (n + 127) // 128  # noqa: E731
    unit = shape.weight_std / FP8_CODE_STD
    out["W_gate_up_s"] = torch.rand((E, blk(2 * I), blk(H)), generator=gen, device=dev,
                                    dtype=torch.float32).add_(0.5).mul_(unit)
    out["W_down_s"] = torch.rand((E, blk(H), blk(I)), generator=gen, device=dev,
                                 dtype=torch.float32).add_(0.5).mul_(unit)
    if shape.bias_kind == "zipf":
        g = ZIPF_GAMMA if gamma is None else gamma
        bias = zipf_bias(E, shape.seed, g).to(dev)
    out["bias"] = bias
    return out


def draw_router_only(shape: LayerShape, device="cpu", gamma: float | None = None) -> dict:
    """x, Wr and bias exactly as draw() produces them, without the expert weights."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(shape.seed)
    out = {
        "x": _normal_bf16((shape.T, shape.H), shape.x_std, gen, dev),
        "Wr": _normal_bf16((shape.E, shape.H), shape.weight_std, gen, dev),
    }
    bias = torch.rand((shape.E,), generator=gen, device=dev, dtype=torch.float32).mul_(0.2).sub_(0.1)
    if shape.bias_kind == "zipf":
        g = ZIPF_GAMMA if gamma is None else gamma
        bias = zipf_bias(shape.E, shape.seed, g).to(dev)
    out["bias"] = bias
    return out


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor (raw bits, no conversion)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def token_sample(T: int, n: int, seed: int) -> torch.Tensor:
    """Sorted, distinct token indices for sampled checks at full size."""
    g = torch.Generator().manual_seed(7919 + seed)
    n = min(n, T)
    return torch.sort(torch.randperm(T, generator=g)[:n]).values


__all__ = ["LayerShape", "WORKLOADS", "draw", "draw_router_only", "zipf_bias", "bf16_bits",
           "token_sample", "ZIPF_GAMMA", "ZIPF_S"]
