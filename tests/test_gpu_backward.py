"""GPU parity of the backward pass (moe_backward) against the oracle's backward.

Both sides differentiate the same routing: the oracle's selected ids and weights (the
GPU forward's routing agrees with them outside near-ties, which the forward tests cover)
are passed to moe_backward. Tolerance: the GPU rounds dy, the pre-activation gradients and
w*h to bf16 before its GEMMs (relative error <= 2^-9 each, independent across elements),
which puts ~1e-3 relative error on a gradient entry; each gradient tensor must be within the
layer's relative-Frobenius bar 1e-2 of the fp64 oracle, and every entry within 2e-2 of the
tensor's largest magnitude.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import rel_fro
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import WORKLOADS, LayerShape, bf16_bits, draw

pytestmark = pytest.mark.gpu

SHAPES = {
    # clips binding, two 128-feature blocks in down, ragged chunks
    "clip": LayerShape("bwd_clip", T=96, H=256, E=6, k=2, I=256, Is=128, limit_routed=0.5, limit_shared=0.25,
                       seed=71, weight_std=0.08),
    # more groups than tokens per group, experts without tokens (zeroed gradients), H = 3 x 128
    "sparse": LayerShape("bwd_sparse", T=40, H=384, E=24, k=2, I=128, Is=256, seed=72, weight_std=0.05),
    # chunks of more than 128 rows (256-row token boxes) and padding to 64 rows, the shared group
    # split in two chunks, no clip, no normalisation
    "big_groups": LayerShape("bwd_big", T=300, H=256, E=3, k=2, I=128, Is=128, scale=2.5,
                             norm_expert_weight=False, seed=73, weight_std=0.05),
    # groups above the 256-row chunk cap (~400 rows per routed group, the shared group in three
    # chunks); k = 2 of 3 experts, so the normalised weights depend on the logits (with k = 1
    # they would be the constant scale and the router-weight gradient exactly zero)
    "huge_groups": LayerShape("bwd_huge", T=600, H=256, E=3, k=2, I=128, Is=256, limit_routed=0.5, seed=74,
                              weight_std=0.05),
    "tiny": WORKLOADS["tiny"],
}


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    _abi.lib()
    yield
    _abi.moe_check_device()


def _gpu_backward(sh, inp, idx, w, dy):
    dev = {k: v.cuda() for k, v in inp.items()}
    d = _abi.desc_of(sh)
    ws = torch.empty(_abi.moe_backward_workspace_size(d), dtype=torch.uint8, device="cuda")
    E, H, I, Is, T = sh.E, sh.H, sh.I, sh.Is, sh.T
    out = {"dx": torch.full((T, H), float("nan"), device="cuda"),
           "dWr": torch.full((E, H), float("nan"), device="cuda"),
           "dW_gate_up": torch.full((E, 2 * I, H), float("nan"), device="cuda"),
           "dW_down": torch.full((E, H, I), float("nan"), device="cuda"),
           "dWsh_gate_up": torch.full((2 * Is, H), float("nan"), device="cuda"),
           "dWsh_down": torch.full((H, Is), float("nan"), device="cuda")}
    _abi.moe_backward(d, dev["x"], dev["Wr"], dev["W_gate_up"], dev["W_down"], dev["Wsh_gate_up"], dev["Wsh_down"],
                      torch.from_numpy(idx).cuda(), torch.from_numpy(w.astype(np.float32)).cuda(),
                      torch.from_numpy(dy).cuda(), out["dx"], out["dWr"], out["dW_gate_up"], out["dW_down"],
                      out["dWsh_gate_up"], out["dWsh_down"], ws)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    return {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("name", list(SHAPES))
def test_backward_matches_oracle(name):
    sh = SHAPES[name]
    inp = draw(sh)
    dy = np.random.default_rng(sh.seed + 1000).standard_normal((sh.T, sh.H)).astype(np.float32)
    ref = oracle.backward(bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(),
                          bf16_bits(inp["W_gate_up"]), bf16_bits(inp["W_down"]), bf16_bits(inp["Wsh_gate_up"]),
                          bf16_bits(inp["Wsh_down"]), dy, k=sh.k, scale=sh.scale, norm=sh.norm_expert_weight,
                          limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    got = _gpu_backward(sh, inp, ref["idx"], ref["w"], dy)
    for key in ("dx", "dWr", "dW_gate_up", "dW_down", "dWsh_gate_up", "dWsh_down"):
        g, r = got[key], ref[key]
        assert np.isfinite(g).all(), f"{key}: unwritten or non-finite entries"
        rf = rel_fro(g, r)
        ma = float(np.abs(g - r).max()) / max(float(np.abs(r).max()), 1e-30)
        print(f"{name} {key}: rel_fro {rf:.2e} max_abs/max {ma:.2e}")
        assert rf <= 1e-2, f"{key} relative Frobenius error {rf:.3e}"
        assert ma <= 2e-2, f"{key} max error {ma:.3e} of the largest entry"
    used = np.unique(ref["idx"])
    unused = np.setdiff1d(np.arange(sh.E), used)
    for e in unused:  # experts without tokens get zero weight gradients
        assert not got["dW_gate_up"][e].any() and not got["dW_down"][e].any() and not got["dWr"][e].any()


@pytest.mark.slow
def test_backward_full_size_one_expert():
    """Step-3.5 prefill shape, forward routing from the GPU: the weight gradients of a
    touched expert with about 8 tokens and the router row of that expert depend only on
    the tokens routed to it, so the oracle's backward over just those tokens gives them
    exactly, with those tokens' dx."""
    sh = WORKLOADS["step35_prefill"]
    inp = draw(sh, device="cuda")
    from sparse_moe_layer_biased_b200.layer import MoeLayer
    _, idx, w = MoeLayer(sh, inp).forward(inp["x"], routing=True)
    dy = torch.randn((sh.T, sh.H), generator=torch.Generator(device="cuda").manual_seed(77), device="cuda")
    d = _abi.desc_of(sh)
    ws = torch.empty(_abi.moe_backward_workspace_size(d), dtype=torch.uint8, device="cuda")
    E, H, I, Is, T = sh.E, sh.H, sh.I, sh.Is, sh.T
    out = {"dx": torch.empty((T, H), device="cuda"), "dWr": torch.empty((E, H), device="cuda"),
           "dW_gate_up": torch.empty((E, 2 * I, H), device="cuda"), "dW_down": torch.empty((E, H, I), device="cuda"),
           "dWsh_gate_up": torch.empty((2 * Is, H), device="cuda"), "dWsh_down": torch.empty((H, Is), device="cuda")}
    _abi.moe_backward(d, inp["x"], inp["Wr"], inp["W_gate_up"], inp["W_down"], inp["Wsh_gate_up"],
                      inp["Wsh_down"], idx, w, dy, out["dx"], out["dWr"], out["dW_gate_up"], out["dW_down"],
                      out["dWsh_gate_up"], out["dWsh_down"], ws)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    idx_h = idx.cpu().numpy()
    counts = np.bincount(idx_h.ravel(), minlength=E)
    e = int(np.where(counts > 0, np.abs(counts - 8), 1 << 30).argmin())  # about 8 tokens: cheap for the oracle
    rows = np.nonzero((idx_h == e).any(1))[0]
    rsel = torch.from_numpy(rows).cuda()
    ref = oracle.backward(bf16_bits(inp["x"][rsel]), bf16_bits(inp["Wr"]), inp["bias"].cpu().numpy(),
                          bf16_bits(inp["W_gate_up"]), bf16_bits(inp["W_down"]), bf16_bits(inp["Wsh_gate_up"]),
                          bf16_bits(inp["Wsh_down"]), dy[rsel].cpu().numpy(), k=sh.k, scale=sh.scale,
                          norm=sh.norm_expert_weight, limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    np.testing.assert_array_equal(np.sort(ref["idx"], 1), np.sort(idx_h[rows], 1))
    pairs = {"dW_gate_up": (out["dW_gate_up"][e], ref["dW_gate_up"][e]), "dW_down": (out["dW_down"][e],
             ref["dW_down"][e]), "dWr": (out["dWr"][e], ref["dWr"][e]), "dx": (out["dx"][rsel], ref["dx"])}
    for key, (g, r) in pairs.items():
        g = g.cpu().numpy()
        rf = rel_fro(g, r)
        ma = float(np.abs(g - r).max()) / max(float(np.abs(r).max()), 1e-30)
        print(f"step35 expert {e} ({len(rows)} tokens) {key}: rel_fro {rf:.2e} max_abs/max {ma:.2e}")
        assert rf <= 1e-2 and ma <= 2e-2, key
