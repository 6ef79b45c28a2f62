"""Pins of the oracle's backward pass (oracle_backward) against torch autograd in float64.

The autograd side restates the forward in torch (fp64 weights, the oracle's selected
expert ids held fixed: no gradient through top-k) and lets autograd differentiate it; the
restatement itself is pinned to the oracle's forward. Shapes keep H, I and Is distinct so a
transposed operand fails, and the cases cover both clips active, no clip, no normalisation
and k = E.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_layer_biased_b200.inputs import LayerShape, bf16_bits, draw

CASES = {
    "clip": LayerShape("bw_clip", T=12, H=48, E=6, k=2, I=16, Is=24, limit_routed=0.3, limit_shared=0.2,
                       seed=61, weight_std=0.3),
    "noclip_nonorm": LayerShape("bw_nonorm", T=10, H=40, E=5, k=3, I=24, Is=8, scale=2.5,
                                norm_expert_weight=False, seed=62, weight_std=0.2),
    "k_equals_E": LayerShape("bw_kE", T=8, H=32, E=4, k=4, I=8, Is=16, limit_routed=0.5, seed=63,
                             weight_std=0.25),
}


def _torch_layer(sh, inp, idx, dy):
    """fp64 restatement of the forward with ids fixed; returns (y, grads by name)."""
    f = lambda t: t.double().clone().requires_grad_(True)  # noqa: E731
    x, Wr = f(inp["x"]), f(inp["Wr"])
    Wgu, Wd = f(inp["W_gate_up"]), f(inp["W_down"])
    Wshgu, Wshd = f(inp["Wsh_gate_up"]), f(inp["Wsh_down"])
    ids = torch.from_numpy(idx).long()
    s = torch.sigmoid(x @ Wr.T)
    sel = torch.gather(s, 1, ids)
    w = sh.scale * sel / sel.sum(1, keepdim=True) if sh.norm_expert_weight else sh.scale * sel

    def mlp(xr, gu, d, L):
        n = gu.shape[0] // 2
        g, u = xr @ gu[:n].T, xr @ gu[n:].T
        a = torch.nn.functional.silu(g)
        if L > 0:
            a, u = torch.clamp(a, max=L), torch.clamp(u, -L, L)
        return (a * u) @ d.T

    y = mlp(x, Wshgu, Wshd, sh.limit_shared)
    for t in range(sh.T):
        for j in range(sh.k):
            e = int(ids[t, j])
            y = y.index_add(0, torch.tensor([t]), w[t, j] * mlp(x[t:t + 1], Wgu[e], Wd[e], sh.limit_routed))
    (y * torch.from_numpy(dy).double()).sum().backward()
    return y.detach().numpy(), {"dx": x.grad, "dWr": Wr.grad, "dW_gate_up": Wgu.grad, "dW_down": Wd.grad,
                                "dWsh_gate_up": Wshgu.grad, "dWsh_down": Wshd.grad}


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_autograd(name):
    sh = CASES[name]
    inp = draw(sh)
    dy = np.random.default_rng(sh.seed).standard_normal((sh.T, sh.H)).astype(np.float32)
    args = (bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), bf16_bits(inp["W_gate_up"]),
            bf16_bits(inp["W_down"]), bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]))
    kw = dict(k=sh.k, scale=sh.scale, norm=sh.norm_expert_weight, limit_routed=sh.limit_routed,
              limit_shared=sh.limit_shared)
    ob = oracle.backward(*args, dy, **kw)
    fw = oracle.forward_full(inp, sh)
    np.testing.assert_array_equal(ob["idx"], fw["idx"])
    y_t, grads = _torch_layer(sh, inp, ob["idx"], dy)
    # the restatement is the oracle's forward (the oracle rounds the logits and scores to fp32)
    np.testing.assert_allclose(y_t, fw["y"], rtol=1e-5, atol=1e-6)
    for key, g in grads.items():
        g = g.numpy()
        scale = np.abs(g).max()
        assert scale > 0, key
        np.testing.assert_allclose(ob[key], g, rtol=1e-5, atol=1e-6 * scale, err_msg=key)
    # dw = dLoss/dw_j = dy . o_j, checked through the chain: dWr is zero on never-selected experts
    never = np.setdiff1d(np.arange(sh.E), np.unique(ob["idx"]))
    assert np.all(ob["dWr"][never] == 0.0)


def test_clips_bind_in_the_clip_case():
    """The clip case exercises both masks (otherwise its pin would not test them)."""
    sh = CASES["clip"]
    inp = draw(sh)
    x = inp["x"].double()
    gu = inp["W_gate_up"].double()
    g = torch.einsum("th,eih->tei", x, gu[:, : sh.I])
    u = torch.einsum("th,eih->tei", x, gu[:, sh.I:])
    a = torch.nn.functional.silu(g)
    assert (a > sh.limit_routed).double().mean() > 0.1
    assert (u.abs() > sh.limit_routed).double().mean() > 0.1


def test_backward_is_linear_in_dy_and_bias_free():
    sh = CASES["clip"]
    inp = draw(sh)
    dy = np.random.default_rng(5).standard_normal((sh.T, sh.H)).astype(np.float32)
    args = (bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), bf16_bits(inp["W_gate_up"]),
            bf16_bits(inp["W_down"]), bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]))
    kw = dict(k=sh.k, scale=sh.scale, norm=True, limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    b1 = oracle.backward(*args, dy, **kw)
    b2 = oracle.backward(*args, 2 * dy, **kw)
    for key in ("dx", "dWr", "dW_gate_up", "dW_down"):
        np.testing.assert_allclose(b2[key], 2 * b1[key], rtol=1e-12, atol=1e-15)
    # a constant bias shift keeps the selection, hence every gradient
    args2 = list(args)
    args2[2] = args[2] + np.float32(0.25)
    b3 = oracle.backward(*args2, dy, **kw)
    for key in ("dx", "dWr", "dW_gate_up", "dW_down", "dWsh_gate_up", "dWsh_down"):
        np.testing.assert_array_equal(b3[key], b1[key])


def test_single_normalised_expert_sends_no_gradient_to_the_router():
    """k = 1 with normalisation: the weight is scale * s / s, the constant scale, so no
    gradient reaches the logits (dWr = 0 and the router part of dx vanishes) while the expert
    weights still get theirs (closed form of the chain rule for this case)."""
    sh = LayerShape("bw_k1", T=9, H=32, E=3, k=1, I=8, Is=16, limit_routed=0.5, seed=64, weight_std=0.25)
    inp = draw(sh)
    dy = np.random.default_rng(sh.seed).standard_normal((sh.T, sh.H)).astype(np.float32)
    ob = oracle.backward(bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), bf16_bits(inp["W_gate_up"]),
                         bf16_bits(inp["W_down"]), bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), dy,
                         k=1, scale=sh.scale, norm=True, limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    assert np.abs(ob["dWr"]).max() <= 1e-12 * max(1.0, np.abs(ob["dW_gate_up"]).max())
    assert np.abs(ob["dW_gate_up"]).max() > 0 and np.abs(ob["dW_down"]).max() > 0
