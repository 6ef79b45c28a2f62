"""The layer call captured in a CUDA graph and replayed.

The library only enqueues work on the caller's stream (no allocation, no synchronisation inside
a call; tensor maps travel as kernel parameters), so a decode loop can capture one call and
replay it with new inputs written into the captured input buffer. Each replay must equal a fresh
eager call on the same input, bit for bit (deterministic mode: no atomic accumulation order), on
the single-CTA, CTA-pair and FP8 paths.
"""
import pytest
import torch

from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import LayerShape, draw, draw_fp8
from sparse_moe_layer_biased_b200.layer import MoeLayer

pytestmark = pytest.mark.gpu

SHAPES = {
    # decode-sized: 32-row chunks on single CTAs (BF16), the FP8 tensor-core kernels (FP8)
    "decode": LayerShape("graph_decode", T=24, H=512, E=40, k=8, I=256, Is=256, limit_routed=0.25, seed=71,
                         weight_std=0.03),
    # prefill-sized with I, Is % 128 == 0 and H % 512 == 0: the CTA-pair kernels (clusters)
    "prefill_pair": LayerShape("graph_prefill", T=600, H=512, E=12, k=4, I=256, Is=256, limit_routed=0.25,
                               seed=72, weight_std=0.03),
}


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    _abi.lib()
    yield
    _abi.moe_check_device()


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_replays_from_a_cuda_graph(name, fp8):
    sh = SHAPES[name]
    inp = (draw_fp8 if fp8 else draw)(sh, device="cuda")
    layer = MoeLayer(sh, inp, deterministic=True)
    x = inp["x"].clone()
    y = torch.empty((sh.T, sh.H), dtype=torch.float32, device="cuda")
    layer.forward(x, y=y)  # eager first: modules loaded and kernel attributes set before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        layer.forward(x, y=y)
    for seed in (1, 2):
        gen = torch.Generator(device="cuda").manual_seed(seed)
        x.copy_(torch.randn(x.shape, generator=gen, device="cuda").to(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        ref = layer.forward(x.clone())
        torch.cuda.synchronize()
        _abi.moe_check_device()
        assert torch.isfinite(y).all()
        assert torch.equal(y, ref), f"replay {seed} differs from the eager call"
    del g
