"""moe_forward_host: batches in host memory, copies overlapped with the forward on the GPU.

Each batch's output must be exactly what moe_forward gives for the same rows on the device
(deterministic mode: a fixed summation order, so equal bit for bit), with page-locked and
with pageable host buffers, for one batch, for more batches than staging buffers, and with
a batch that reuses a staging buffer while its previous output is still being copied out.
"""
import numpy as np
import pytest
import torch

from _parity import check_output
import oracle
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import WORKLOADS, LayerShape, draw, draw_fp8
from sparse_moe_layer_biased_b200.layer import MoeLayer

pytestmark = pytest.mark.gpu

SHAPE = LayerShape("host_pipe", T=300, H=512, E=12, k=4, I=256, Is=256, limit_routed=0.25, limit_shared=0.125,
                   seed=81)


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    _abi.lib()
    yield
    _abi.moe_check_device()


def _batches(sh, n):
    return torch.stack([draw(sh.replace(seed=sh.seed + 10 * i))["x"] for i in range(n)])


@pytest.mark.parametrize("n,pinned", [(1, True), (5, True), (3, False)])
def test_forward_host_equals_device_forward(n, pinned):
    sh = SHAPE
    dev = {k: v.cuda() for k, v in draw(sh).items()}
    layer = MoeLayer(sh, dev, deterministic=True)
    xs = _batches(sh, n)
    x_host = xs.pin_memory() if pinned else xs.clone()
    y_host = torch.full((n, sh.T, sh.H), float("nan"), dtype=torch.float32)
    if pinned:
        y_host = y_host.pin_memory()
    layer.forward_host(x_host, y_host)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    for i in range(n):
        y_dev = layer.forward(xs[i].cuda())
        torch.cuda.synchronize()
        assert torch.equal(y_host[i], y_dev.cpu()), f"batch {i}"


def test_forward_host_against_oracle():
    sh = WORKLOADS["tiny"]
    inp = draw(sh)
    layer = MoeLayer(sh, {k: v.cuda() for k, v in inp.items()})
    y = layer.forward_host(inp["x"][None].pin_memory())
    torch.cuda.synchronize()
    ref = oracle.forward_full(inp, sh)
    keep = ref["margin"] >= 1e-6  # near-tied selections are excluded as in the layer's parity tests
    check_output(y[0].numpy()[keep], ref["y"][keep], "tiny host")


def test_forward_host_fp8_equals_device_forward():
    sh = SHAPE.replace(name="host_pipe_fp8", weight_std=0.03)
    layer = MoeLayer(sh, {k: v.cuda() for k, v in draw_fp8(sh).items()}, deterministic=True)
    assert layer.fp8
    xs = _batches(sh, 3)
    y_host = layer.forward_host(xs.pin_memory())
    torch.cuda.synchronize()
    _abi.moe_check_device()
    for i in range(3):
        y_dev = layer.forward(xs[i].cuda())
        torch.cuda.synchronize()
        assert torch.equal(y_host[i], y_dev.cpu()), f"batch {i}"
