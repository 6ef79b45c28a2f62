"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test ties one part of the oracle to a hand-derived example, a closed form,
an invariant of the method, a textbook routine or brute force, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand, bias
leaking into the weights, gate and up swapped) fails at least one of them.

Method: "MAX 中 Step-3.5-Flash 架构解析", sections "MoE共享专家、sigmoid 路由与激活裁剪"
and "Step3p5Config配置项全解".
"""
import json
import os

import numpy as np
import pytest
import scipy.special
import torch

from sparse_moe_layer_biased_b200.inputs import WORKLOADS, LayerShape, bf16_bits, draw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


def _bits(a):
    return bf16_bits(torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def _hand_layer(g):
    sh = g["shape"]
    H, E, I, Is = sh["H"], sh["E"], sh["I"], sh["Is"]
    W = g["weights"]
    Wr = np.zeros((E, H), np.float32)
    Wr[:, 0] = W["Wr_col0"]
    Wgu = np.zeros((E, 2 * I, H), np.float32)
    Wd = np.zeros((E, H, I), np.float32)
    for e in range(E):
        Wgu[e, :I, 0] = W["W_gate_up_col0"][str(e)]["gate"]
        Wgu[e, I:, 0] = W["W_gate_up_col0"][str(e)]["up"]
        Wd[e] = np.asarray(W["W_down"][str(e)], np.float32)
    Wsh_gu = np.zeros((2 * Is, H), np.float32)
    Wsh_gu[:Is, 0] = W["Wsh_gate_up_col0"]["gate"]
    Wsh_gu[Is:, 0] = W["Wsh_gate_up_col0"]["up"]
    Wsh_d = np.asarray(W["Wsh_down"], np.float32)
    return Wr, Wgu, Wd, Wsh_gu, Wsh_d


@pytest.mark.parametrize("case", [0, 1])
def test_hand_example(oracle_mod, case):
    g = json.load(open(GOLDEN))
    Wr, Wgu, Wd, Wsh_gu, Wsh_d = _hand_layer(g)
    c = g["cases"][case]
    x = np.asarray([c["x"]], np.float32)
    bias = np.asarray(c["bias"], np.float32)
    k = g["shape"]["k"]
    r = oracle_mod.router(_bits(x), _bits(Wr), bias, k)
    exp = c["expected"]
    assert r["idx"][0].tolist() == exp["ids"]
    np.testing.assert_allclose(r["w"][0], exp["weights"], rtol=1e-6)
    if "margin" in exp:
        np.testing.assert_allclose(r["margin"][0], exp["margin"], rtol=1e-6)
    else:
        m = (np.float32(0.5) + np.float32(0.3)) - (np.float32(0.5) + np.float32(0.1))
        assert r["margin"][0] == np.float32(m)
    experts = {e: (_bits(Wgu[e]), _bits(Wd[e])) for e in range(g["shape"]["E"])}
    for lim, key in [(0.0, "y_limit0"), (1.5, "y_limit1.5")]:
        out = oracle_mod.forward_tokens(_bits(x), _bits(Wr), bias, experts, _bits(Wsh_gu), _bits(Wsh_d),
                                        k=k, limit_routed=lim, limit_shared=0.0)
        np.testing.assert_allclose(out["y"][0], exp[key], rtol=1e-6, atol=1e-12)


def _rand_router(T, H, E, seed, std=0.05):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    Wr = (torch.randn((E, H), generator=g) * std).to(torch.bfloat16)
    bias = (torch.rand((E,), generator=g) * 0.2 - 0.1).float()
    return bf16_bits(x), bf16_bits(Wr), bias.numpy()


def _brute_select(b, s, k, scale=3.0):
    """Full sort of every expert by (b desc, index asc); weights 3 s / sum s."""
    E = b.shape[0]
    order = sorted(range(E), key=lambda e: (-float(b[e]), e))
    ids = order[:k]
    ss = np.asarray([float(s[e]) for e in ids])
    return ids, scale * ss / ss.sum()


def test_router_logits_match_library_matmul(oracle_mod):
    x, Wr, _ = _rand_router(37, 96, 11, seed=1)
    xf = x.astype(np.uint32) << 16
    wf = Wr.astype(np.uint32) << 16
    ref = (xf.view(np.float32).astype(np.float64) @ wf.view(np.float32).astype(np.float64).T)
    got = oracle_mod.router_logits(x, Wr)
    # double accumulation, one fp32 rounding: within 1 fp32 ulp of the fp64 product
    np.testing.assert_allclose(got, ref.astype(np.float32), rtol=1.2e-7, atol=1e-30)


def test_router_selection_brute_force(oracle_mod):
    for seed, (T, H, E, k) in enumerate([(40, 64, 12, 3), (25, 128, 16, 4), (9, 64, 33, 8), (5, 64, 8, 8)]):
        x, Wr, bias = _rand_router(T, H, E, seed + 10)
        r = oracle_mod.router(x, Wr, bias, k)
        s = scipy.special.expit(r["logits"].astype(np.float64)).astype(np.float32)
        np.testing.assert_allclose(r["scores"], s, rtol=2.4e-7)  # textbook sigmoid, fp32 result
        for t in range(T):
            b = (r["scores"][t] + bias).astype(np.float32)
            ids, w = _brute_select(b, r["scores"][t], k)
            assert r["idx"][t].tolist() == ids
            np.testing.assert_allclose(r["w"][t], w, rtol=1e-14)


def test_weights_sum_to_scale(oracle_mod):
    sh = WORKLOADS["tiny"]
    inp = draw(sh)
    r = oracle_mod.router(bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), sh.k)
    ulp3 = np.spacing(np.float32(3.0))
    assert np.all(np.abs(r["w32"].astype(np.float64).sum(1) - 3.0) <= 8 * ulp3)
    assert np.all(np.abs(r["w"].sum(1) - 3.0) <= 1e-12)
    # without normalisation the weight is scale * s of the selected expert
    r2 = oracle_mod.router(bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), sh.k, norm=False)
    sel_s = np.take_along_axis(r2["scores"], r2["idx"].astype(np.int64), 1)
    np.testing.assert_array_equal(r2["w"], 3.0 * sel_s.astype(np.float64))


def test_bias_shift_keeps_selection_and_weights(oracle_mod):
    x, Wr, bias = _rand_router(64, 128, 24, seed=3)
    r0 = oracle_mod.router(x, Wr, bias, 6)
    r1 = oracle_mod.router(x, Wr, (bias + np.float32(0.125)).astype(np.float32), 6)
    ok = r0["margin"] > 1e-6
    assert ok.sum() > 50
    np.testing.assert_array_equal(r0["idx"][ok], r1["idx"][ok])
    np.testing.assert_array_equal(r0["w"][ok], r1["w"][ok])


def test_bias_changes_selection_not_weights(oracle_mod):
    T, E, k = 32, 20, 4
    x, Wr, _ = _rand_router(T, 64, E, seed=4)
    forced = [17, 2, 11, 5]
    bias = np.zeros(E, np.float32)
    bias[forced] = 10.0
    r = oracle_mod.router(x, Wr, bias, k)
    for t in range(T):
        s = r["scores"][t]
        want = sorted(forced, key=lambda e: (-float(s[e] + np.float32(10.0)), e))
        assert r["idx"][t].tolist() == want
        ss = s[want].astype(np.float64)
        np.testing.assert_allclose(r["w"][t], 3.0 * ss / ss.sum(), rtol=1e-14)
    # without the bias the same tokens mostly pick other experts
    r0 = oracle_mod.router(x, Wr, np.zeros(E, np.float32), k)
    assert (np.sort(r0["idx"], 1) != np.sort(np.asarray(forced))).any()


def test_k_equals_E(oracle_mod):
    x, Wr, bias = _rand_router(16, 64, 6, seed=5)
    r = oracle_mod.router(x, Wr, bias, 6)
    assert np.all(np.sort(r["idx"], 1) == np.arange(6))
    np.testing.assert_allclose(np.take_along_axis(r["w"], np.argsort(r["idx"], 1), 1),
                               3.0 * r["scores"].astype(np.float64)
                               / r["scores"].astype(np.float64).sum(1, keepdims=True),
                               rtol=1e-14)
    assert np.all(np.isinf(r["margin"]))


def test_nan_routing_stays_in_range(oracle_mod):
    x, Wr, bias = _rand_router(8, 64, 10, seed=6)
    x = x.copy()
    x[2, 5] = 0x7FC0  # bf16 NaN
    r = oracle_mod.router(x, Wr, bias, 3)
    assert np.all((r["idx"] >= 0) & (r["idx"] < 10))
    assert all(len(set(row)) == 3 for row in r["idx"].tolist())
    assert r["idx"][2].tolist() == [0, 1, 2]  # every biased score NaN: ties by index


def test_underflowed_scores_give_scale_over_k(oracle_mod):
    logits = np.full((3, 5), -200.0, np.float32)
    r = oracle_mod.router_select(logits, np.zeros(5, np.float32), 2)
    assert np.all(r["scores"] == 0)
    np.testing.assert_array_equal(r["w"], 1.5)
    assert r["idx"].tolist() == [[0, 1]] * 3


def test_permute_brute_force(oracle_mod):
    rng = np.random.default_rng(0)
    cases = []
    T, E, k = 50, 9, 3
    cases.append((np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32), E))
    # skewed: every token picks expert 0 first; experts 7, 8 stay empty
    idx = np.stack([np.concatenate([[0], 1 + rng.permutation(6)[: k - 1]]) for _ in range(T)]).astype(np.int32)
    cases.append((idx, E))
    cases.append((np.zeros((0, 2), np.int32), 4))
    for idx, E in cases:
        T, k = idx.shape
        p = oracle_mod.permute(idx, E)
        np.testing.assert_array_equal(p["counts"][:E], np.bincount(idx.ravel(), minlength=E))
        assert p["counts"][E] == T
        np.testing.assert_array_equal(p["offsets"], np.concatenate([[0], np.cumsum(p["counts"])]))
        entries = sorted((int(idx[t, j]), t, j) for t in range(T) for j in range(k))
        for slot, (e, t, j) in enumerate(entries):
            assert p["slot_of"][t, j] == slot
            assert p["perm_token"][slot] == t
        np.testing.assert_array_equal(p["perm_token"][T * k:], np.arange(T))


def _swiglu_textbook(x, Wgu, Wd, limit):
    """Two-matmul SwiGLU MLP in fp64 torch (F.silu), gate rows first."""
    I = Wgu.shape[0] // 2
    g = x @ Wgu[:I].T
    u = x @ Wgu[I:].T
    a = torch.nn.functional.silu(g)
    if limit > 0:
        a = torch.clamp(a, max=limit)
        u = torch.clamp(u, -limit, limit)
    return (a * u) @ Wd.T


def test_single_expert_reduces_to_textbook_mlp(oracle_mod):
    sh = LayerShape("one", T=12, H=64, E=1, k=1, I=32, Is=48, seed=9, weight_std=0.1)
    inp = draw(sh)
    for lim in (0.0, 0.25):  # limits are fp32 in the layer description: use fp32-exact values
        out = oracle_mod.forward_full(inp, sh, limit_routed=lim, limit_shared=0.125)
        f64 = {k: v.double() for k, v in inp.items()}
        ref = 3.0 * _swiglu_textbook(f64["x"], f64["W_gate_up"][0], f64["W_down"][0], lim)
        ref = ref + _swiglu_textbook(f64["x"], f64["Wsh_gate_up"], f64["Wsh_down"], 0.125)
        np.testing.assert_allclose(out["y"], ref.numpy(), rtol=1e-10, atol=1e-13)
        np.testing.assert_array_equal(out["w"], 3.0)


@pytest.mark.parametrize("shape", [WORKLOADS["tiny"],
                                   LayerShape("odd", T=19, H=128, E=7, k=3, I=64, Is=192, seed=11,
                                              limit_routed=0.05, limit_shared=0.04, weight_std=0.05)])
def test_sparse_equals_dense_brute_force(oracle_mod, shape):
    inp = draw(shape)
    y = oracle_mod.forward_full(inp, shape)["y"]
    yd = oracle_mod.forward_dense(
        bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), bf16_bits(inp["W_gate_up"]),
        bf16_bits(inp["W_down"]), bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), k=shape.k,
        limit_routed=shape.limit_routed, limit_shared=shape.limit_shared)
    np.testing.assert_allclose(y, yd, rtol=1e-12, atol=1e-15)


def test_limit_zero_means_no_clip(oracle_mod):
    sh = WORKLOADS["tiny"].replace(weight_std=0.2)
    inp = draw(sh)
    y0 = oracle_mod.forward_full(inp, sh, limit_routed=0.0, limit_shared=0.0)["y"]
    yinf = oracle_mod.forward_full(inp, sh, limit_routed=1e30, limit_shared=1e30)["y"]
    np.testing.assert_array_equal(y0, yinf)
    y7 = oracle_mod.forward_full(inp, sh, limit_routed=0.5, limit_shared=0.0)["y"]
    assert np.abs(y7 - y0).max() > 1e-3


def test_clip_matches_elementwise_and_bites(oracle_mod):
    sh = WORKLOADS["tiny"].replace(weight_std=0.2)
    inp = draw(sh)
    L = 0.5
    x = inp["x"].double().numpy()
    clipped = total = 0
    for e in range(3):
        Wgu = inp["W_gate_up"][e].double().numpy()
        g = x[:8] @ Wgu[: sh.I].T
        u = x[:8] @ Wgu[sh.I:].T
        a = g * scipy.special.expit(g)
        ref = np.minimum(a, L) * np.clip(u, -L, L)
        clipped += int(((a > L) | (np.abs(u) > L)).sum())
        total += a.size
        for t in range(8):
            got = oracle_mod.swiglu_hidden(bf16_bits(inp["x"][t]), bf16_bits(inp["W_gate_up"][e]), L)
            np.testing.assert_allclose(got, ref[t], rtol=1e-12, atol=1e-14)
    assert clipped / total >= 0.2


def test_token_permutation_equivariance(oracle_mod):
    sh = WORKLOADS["tiny"]
    inp = draw(sh)
    perm = torch.randperm(sh.T, generator=torch.Generator().manual_seed(5))
    out = oracle_mod.forward_full(inp, sh)
    inp2 = dict(inp)
    inp2["x"] = inp["x"][perm]
    out2 = oracle_mod.forward_full(inp2, sh)
    np.testing.assert_array_equal(out2["y"], out["y"][perm.numpy()])
    np.testing.assert_array_equal(out2["idx"], out["idx"][perm.numpy()])


def test_scale_is_linear_without_normalisation(oracle_mod):
    sh = WORKLOADS["tiny"].replace(norm_expert_weight=False)
    inp = draw(sh)
    ya = oracle_mod.forward_full(inp, sh, scale=1.0)["y"]
    yb = oracle_mod.forward_full(inp, sh, scale=3.0)["y"]
    zero = dict(inp)
    zero["W_gate_up"] = torch.zeros_like(inp["W_gate_up"])
    ysh = oracle_mod.forward_full(zero, sh, scale=1.0)["y"]  # shared expert alone
    np.testing.assert_allclose(yb - ysh, 3.0 * (ya - ysh), rtol=1e-9, atol=1e-15)


def test_zipf_recipe_reaches_target_share(oracle_mod):
    from sparse_moe_layer_biased_b200 import inputs

    sh = WORKLOADS["step5_skewed"].replace(T=1024)
    r = inputs.draw_router_only(sh)
    sel = oracle_mod.router(bf16_bits(r["x"]), bf16_bits(r["Wr"]), r["bias"].numpy(), sh.k)
    counts = np.sort(np.bincount(sel["idx"].ravel(), minlength=sh.E))[::-1]
    share = counts[:8].sum() / counts.sum()
    assert 0.26 <= share <= 0.34
    assert counts[0] / counts.sum() <= 1.0 / sh.k


def test_given_routing_reproduces_the_router_path(oracle_mod):
    """With the oracle router's own ids and weights, the given-routing forward is the
    routed forward; with duplicated ids the expert output is added once per slot."""
    sh = LayerShape("gr", T=21, H=128, E=9, k=3, I=64, Is=128, seed=31, limit_routed=0.25, weight_std=0.05)
    inp = draw(sh)
    full = oracle_mod.forward_full(inp, sh)
    gu, d = bf16_bits(inp["W_gate_up"]), bf16_bits(inp["W_down"])
    experts = {e: (gu[e], d[e]) for e in range(sh.E)}
    y = oracle_mod.forward_given_routing(bf16_bits(inp["x"]), full["idx"], full["w"].astype(np.float32), experts,
                                         bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), E=sh.E,
                                         limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    # weights pass through fp32 here (the replay interface is fp32): relative 6e-8 per weight
    np.testing.assert_allclose(y, full["y"], rtol=1e-6, atol=1e-7 * np.abs(full["y"]).max())
    dup = np.full((sh.T, 2), 4, np.int32)
    w = np.full((sh.T, 2), 0.5, np.float32)
    y2 = oracle_mod.forward_given_routing(bf16_bits(inp["x"]), dup, w, experts, bf16_bits(inp["Wsh_gate_up"]),
                                          bf16_bits(inp["Wsh_down"]), E=sh.E, limit_routed=sh.limit_routed,
                                          limit_shared=sh.limit_shared)
    one = oracle_mod.forward_given_routing(bf16_bits(inp["x"]), dup[:, :1], np.ones((sh.T, 1), np.float32), experts,
                                           bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), E=sh.E,
                                           limit_routed=sh.limit_routed, limit_shared=sh.limit_shared)
    np.testing.assert_allclose(y2, one, rtol=1e-12, atol=1e-15)
