"""The E4M3 hi/lo split of the token operand used by the FP8 tensor-core decode kernels.

The kernels scale each token row so its largest magnitude lies in [2^6, 2^7), multiply by a
block scale factor in [2^-1, 2) (so |v| < 2^8, inside E4M3's range of 448), round v to fp16
and split it into hi = e4m3(v) and lo = e4m3(v - hi). The kernels' comments and the design
notes claim hi + lo keeps v to about 2^-8 relative (2^-10 absolute where v - hi falls below
E4M3's normal range), the precision of a bf16 operand. These checks pin that claim with
torch's own fp16 and float8_e4m3fn roundings (round to nearest even, as the PTX conversions
the kernels use), independent of the GPU code.
"""
import torch

F8 = torch.float8_e4m3fn


def split(v: torch.Tensor):
    v16 = v.to(torch.float16)
    hi = v16.float().to(F8)
    r = (v16.float() - hi.float()).to(torch.float16)  # exact in fp16
    lo = r.float().to(F8)
    return v16, hi, r, lo


def test_residual_is_exact_in_fp16():
    g = torch.Generator().manual_seed(0)
    v = (torch.rand(200000, generator=g) * 2 - 1) * 255.0
    v16, hi, r, _ = split(v)
    assert torch.equal(r.double(), v16.double() - hi.double())


def test_hi_lo_relative_error_bound():
    """|v - (hi + lo)| <= 2^-8 |v| + 2^-10 for |v| < 2^8 (fp16 rounding of v included)."""
    g = torch.Generator().manual_seed(1)
    mags = torch.exp2(torch.rand(400000, generator=g) * 20 - 12)  # 2^-12 .. 2^8
    v = torch.where(torch.rand(400000, generator=g) < 0.5, -mags, mags).clamp(-255.9, 255.9)
    _, hi, _, lo = split(v)
    err = (v.double() - (hi.double() + lo.double())).abs()
    assert torch.all(err <= v.double().abs() * 2.0 ** -8 + 2.0 ** -10)
    # typical values of a scaled row (|v| in [2^3, 2^8)) carry about 8 significant bits
    big = v.abs() >= 8
    rel = (err[big] / v.double().abs()[big])
    assert rel.max() <= 2.0 ** -8 and rel.mean() <= 2.0 ** -10


def test_single_e4m3_operand_would_miss_the_layer_bar():
    """Without lo, one E4M3 rounding leaves a relative error of up to 2^-4: a dot product of
    random-sign terms inherits its size (||v - hi|| / ||v|| about 2-3%), above the layer's 1e-2
    bar; with lo it drops below 1e-3 (values of a row scaled to a largest magnitude of 2^7)."""
    g = torch.Generator().manual_seed(2)
    v = torch.randn(100000, generator=g) * 30
    _, hi, _, lo = split(v)
    vd = v.double()
    rel_hi = (vd - hi.double()).norm() / vd.norm()
    rel_hl = (vd - hi.double() - lo.double()).norm() / vd.norm()
    assert rel_hi > 1e-2 and rel_hl < 1e-3
