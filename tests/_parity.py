"""Comparison helpers shared by the GPU parity tests.

Tolerances (fixed by the layer's acceptance bar): expert ids and per-expert counts
bit-exact except tokens whose oracle margin between the k-th and (k+1)-th biased score
is below 1e-6 (reported and excluded, like near-tied selections in the Step-5-Preview
forward-parity table); outputs within relative Frobenius error 1e-2 and max abs error
3e-2 of the fp64 oracle.
"""
import numpy as np
import torch

import oracle
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import bf16_bits

NEAR_TIE = 1e-6
REL_FRO = 1e-2
MAX_ABS = 3e-2
# Routing weights: the GPU accumulates the fp32 logits over H = 4096 products in another
# order than the oracle (one rounding of an fp64 sum); the logit difference reaches a few
# 1e-6 and passes into s and w = 3 s / sum(s) with a factor <= 1, so 2e-5 relative.
W_RTOL = 2e-5


def rel_fro(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def gpu_router(shape, inp, T=None):
    T = shape.T if T is None else T
    dev = inp["x"].device
    idx = torch.empty((T, shape.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, shape.k), dtype=torch.float32, device=dev)
    margin = torch.empty((T,), dtype=torch.float32, device=dev)
    _abi.moe_router(_abi.desc_of(shape, T=T), inp["x"], inp["Wr"], inp["bias"], idx, w, margin)
    torch.cuda.synchronize()
    return {"idx": idx.cpu().numpy(), "w": w.cpu().numpy(), "margin": margin.cpu().numpy()}


def oracle_router(shape, inp, rows=None):
    x = inp["x"] if rows is None else inp["x"][rows]
    return oracle.router(bf16_bits(x), bf16_bits(inp["Wr"]), inp["bias"].cpu().numpy(), shape.k, shape.scale,
                         shape.norm_expert_weight)


def check_routing(g_idx, g_w, o, E, k):
    """Bit-exact id sets and per-expert counts outside near-ties; weights within W_RTOL.

    Returns the boolean mask of compared (non-excluded) tokens.
    """
    keep = o["margin"] >= NEAR_TIE  # NaN margins compare False: excluded
    g_sorted = np.sort(g_idx, 1)
    o_sorted = np.sort(o["idx"], 1)
    bad = np.nonzero(keep & (g_sorted != o_sorted).any(1))[0]
    assert bad.size == 0, f"routing differs on {bad.size} tokens, e.g. {bad[:5]} margins {o['margin'][bad[:5]]}"
    assert np.all((g_idx >= 0) & (g_idx < E))
    gc = np.bincount(g_idx[keep].ravel(), minlength=E)
    oc = np.bincount(o["idx"][keep].ravel(), minlength=E)
    np.testing.assert_array_equal(gc, oc)
    # weights compared per expert id (rank order may differ only inside near-ties)
    go = np.argsort(g_idx, 1, kind="stable")
    oo = np.argsort(o["idx"], 1, kind="stable")
    gw = np.take_along_axis(g_w, go, 1)[keep]
    ow = np.take_along_axis(o["w"], oo, 1)[keep]
    np.testing.assert_allclose(gw, ow, rtol=W_RTOL, atol=1e-7)
    return keep


def check_output(y_gpu, y_ref, what=""):
    rf = rel_fro(y_gpu, y_ref)
    ma = float(np.max(np.abs(np.asarray(y_gpu, np.float64) - y_ref))) if y_ref.size else 0.0
    assert rf <= REL_FRO, f"{what} relative Frobenius error {rf:.3e}"
    assert ma <= MAX_ABS, f"{what} max abs error {ma:.3e}"
    return rf, ma


def host_experts(inp, ids):
    """Host copies of the W_gate_up / W_down slices of the given expert ids."""
    ids = sorted(set(int(e) for e in np.asarray(ids).ravel()))
    gu = inp["W_gate_up"]
    d = inp["W_down"]
    return {e: (bf16_bits(gu[e]), bf16_bits(d[e])) for e in ids}


def oracle_forward_rows(shape, inp, rows):
    """Oracle layer output for the listed token rows (only their experts are copied)."""
    x_rows = inp["x"][rows]
    r = oracle.router(bf16_bits(x_rows), bf16_bits(inp["Wr"]), inp["bias"].cpu().numpy(), shape.k, shape.scale,
                      shape.norm_expert_weight)
    experts = host_experts(inp, r["idx"])
    return oracle.forward_tokens(bf16_bits(x_rows), bf16_bits(inp["Wr"]), inp["bias"].cpu().numpy(), experts,
                                 bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), k=shape.k,
                                 scale=shape.scale, norm=shape.norm_expert_weight,
                                 limit_routed=shape.limit_routed, limit_shared=shape.limit_shared)
