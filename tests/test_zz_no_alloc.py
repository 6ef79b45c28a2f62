"""moe_forward_noalloc: the whole layer on the library's built-in 16 MiB scratch.

Some callers cannot allocate device memory when they run the layer: a serving runtime
that gave nearly all device memory to a fixed pool at start-up, a decode loop that must
not risk the device synchronisation of cudaMalloc / cudaFree, or a plugin that has no
access to its host framework's allocator. For them the library carries its own scratch
array and the caller passes only inputs and outputs.

The GPU test makes two calls in a row through the C ABI, on two different inputs, and
checks each against moe_forward with a caller-allocated workspace: the same routing, the
output within the layer's tolerance (relative Frobenius 1e-2, max abs 3e-2), and bit-equal
output in the deterministic mode, where both run the same kernels in the same order.
This file sorts last so a run that stops at the first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import WORKLOADS, draw

REL_FRO = 1e-2
MAX_ABS = 3e-2
FAKE = 1 << 20  # never dereferenced: the size check fails first


def test_noalloc_rejects_calls_larger_than_its_scratch():
    L = _abi.lib()
    big = _abi.desc_of(WORKLOADS["step35_prefill"])  # needs ~347 MiB of workspace
    args = [FAKE] * 8
    assert L.moe_forward_noalloc(ctypes.byref(big), *args, None, None, None) == 3
    limit = _abi.desc_of(WORKLOADS["step35_decode"], T=189)  # first token count above 16 MiB
    assert L.moe_forward_noalloc(ctypes.byref(limit), *args, None, None, None) == 3
    empty = _abi.desc_of(WORKLOADS["step35_decode"], T=0)
    assert L.moe_forward_noalloc(ctypes.byref(empty), None, None, None, None, None, None, None, None, None,
                                 None, None) == 0


def test_noalloc_token_limits_fit_the_scratch():
    """The documented limits at H = 4096, E = 288, k = 8, I = Is = 1280: 188 tokens fit the
    16 MiB scratch and 189 do not in the default mode; 70 and 71 in the deterministic mode."""
    sh = WORKLOADS["step35_decode"]
    for det, last in ((False, 188), (True, 70)):
        assert _abi.moe_workspace_size(_abi.desc_of(sh, T=last, deterministic=det)) <= 16 << 20
        assert _abi.moe_workspace_size(_abi.desc_of(sh, T=last + 1, deterministic=det)) > 16 << 20
    L = _abi.lib()
    args = [FAKE] * 8
    over = _abi.desc_of(sh, T=71, deterministic=True)
    assert L.moe_forward_noalloc(ctypes.byref(over), *args, None, None, None) == 3


def _forward_with_workspace(d, inp, x):
    T, H, k = x.shape[0], inp["Wr"].shape[1], d.k
    ws = torch.empty(_abi.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    _abi.moe_forward(d, x, inp["Wr"], inp["bias"], inp["W_gate_up"], inp["W_down"], inp["Wsh_gate_up"],
                     inp["Wsh_down"], y, ws, idx, w)
    return y, idx, w


def _forward_noalloc(d, inp, x):
    T, H, k = x.shape[0], inp["Wr"].shape[1], d.k
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    _abi.moe_forward_noalloc(d, x, inp["Wr"], inp["bias"], inp["W_gate_up"], inp["W_down"], inp["Wsh_gate_up"],
                             inp["Wsh_down"], y, idx, w)
    return y, idx, w


@pytest.mark.gpu
@pytest.mark.parametrize("deterministic", [False, True])
def test_noalloc_matches_forward_on_two_calls_in_a_row(deterministic):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    shape = WORKLOADS["step35_decode"]  # decode-sized call: T = 64, H = 4096, E = 288, k = 8
    inp = draw(shape, device="cuda")
    d = _abi.desc_of(shape, deterministic=deterministic)
    g = torch.Generator(device="cuda").manual_seed(1234)
    second_x = torch.randn((shape.T, shape.H), generator=g, device="cuda").to(torch.bfloat16)
    for x in (inp["x"], second_x):  # two calls in a row, different inputs
        y_na, idx_na, w_na = _forward_noalloc(d, inp, x)
        y_ws, idx_ws, w_ws = _forward_with_workspace(d, inp, x)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx_na.cpu().numpy(), idx_ws.cpu().numpy())
        np.testing.assert_array_equal(w_na.cpu().numpy(), w_ws.cpu().numpy())
        a = y_na.double().cpu().numpy()
        b = y_ws.double().cpu().numpy()
        assert np.isfinite(a).all()
        assert np.linalg.norm(a - b) / np.linalg.norm(b) <= REL_FRO
        assert np.abs(a - b).max() <= MAX_ABS
        if deterministic:
            np.testing.assert_array_equal(a, b)
    _abi.moe_check_device()
