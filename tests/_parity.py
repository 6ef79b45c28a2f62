"""Comparison helpers shared by the GPU parity tests.

Tolerances (fixed by the layer's acceptance bar): expert ids and per-expert counts
bit-exact except tokens whose oracle margin between the k-th and (k+1)-th biased score
is below 1e-6 (reported and excluded from the bit-exact comparison, like near-tied
selections in the Step-5-Preview forward-parity table); outputs within relative Frobenius
error 1e-2 and max abs error 3e-2 of the fp64 oracle.

Near-tie tokens are not left unchecked: check_near_ties verifies that the GPU's set
differs from the oracle's only by swaps among experts whose biased score lies within 1e-6
of the oracle's k-th, and that its weights are the normalised scaled scores of its own
set; check_near_tie_outputs compares their outputs with the oracle's given-routing
forward on the GPU's own ids and weights.
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


def near_tie_tokens(o):
    """Tokens excluded from the bit-exact comparison whose margin is a number (NaN rows,
    where every biased score is NaN, are checked for in-range ids only)."""
    m = o["margin"]
    return np.nonzero(np.isfinite(m) & (m < NEAR_TIE))[0]


def check_near_ties(shape, inp, g_idx, g_w, o, rows=None):
    """The GPU's choice on every near-tie token is a valid top-k: it equals the oracle's set
    except for swaps among experts whose biased score (oracle's s + bias, fp32) lies within
    NEAR_TIE of the oracle's k-th biased score, and its weights are scale * s / sum(s) over
    its own set (scale * s without normalisation), from the oracle's scores. `rows` maps
    positions of g_idx / o to token rows of inp["x"] (default: identity). Returns the
    number of tokens validated."""
    ties = near_tie_tokens(o)
    if ties.size == 0:
        return 0
    xrows = ties if rows is None else np.asarray(rows)[ties]
    bias = inp["bias"].cpu().numpy().astype(np.float32)
    r = oracle.router(bf16_bits(inp["x"][torch.as_tensor(xrows, device=inp["x"].device)]),
                      bf16_bits(inp["Wr"]), bias, shape.k, shape.scale, shape.norm_expert_weight)
    s = r["scores"]
    b = (s + bias[None, :]).astype(np.float32)
    for i, t in enumerate(ties):
        O = [int(e) for e in o["idx"][t]]
        G = [int(e) for e in g_idx[t]]
        assert len(set(G)) == shape.k and all(0 <= e < shape.E for e in G), f"token {t}: ids {G}"
        bk = min(float(b[i, e]) for e in O)  # the oracle's k-th biased score
        for e in set(G) - set(O):
            assert b[i, e] >= bk - NEAR_TIE, f"token {t}: expert {e} is not tied with the k-th ({b[i, e]} vs {bk})"
        for e in set(O) - set(G):
            assert b[i, e] <= bk + NEAR_TIE, f"token {t}: dropped expert {e} is not tied ({b[i, e]} vs {bk})"
        sg = s[i, G].astype(np.float64)
        expect = shape.scale * sg / sg.sum() if shape.norm_expert_weight else shape.scale * sg
        np.testing.assert_allclose(g_w[t], expect, rtol=W_RTOL, atol=1e-7, err_msg=f"token {t}")
    return int(ties.size)


def check_near_tie_outputs(shape, inp, y_rows, g_idx, g_w, o, rows=None):
    """Outputs of the near-tie tokens against the oracle's forward for the GPU's own ids and
    weights (same bar as every other token). y_rows / g_idx / g_w / o are indexed like
    check_near_ties. Returns the number of tokens compared."""
    ties = near_tie_tokens(o)
    if ties.size == 0:
        return 0
    xrows = ties if rows is None else np.asarray(rows)[ties]
    ids = np.ascontiguousarray(g_idx[ties], np.int32)
    ref = oracle.forward_given_routing(
        bf16_bits(inp["x"][torch.as_tensor(xrows, device=inp["x"].device)]), ids,
        np.ascontiguousarray(g_w[ties], np.float32), host_experts(inp, ids), bf16_bits(inp["Wsh_gate_up"]),
        bf16_bits(inp["Wsh_down"]), E=shape.E, limit_routed=shape.limit_routed, limit_shared=shape.limit_shared)
    check_output(np.asarray(y_rows)[ties], ref, f"{shape.name} near-tie tokens")
    return int(ties.size)


def chunk_bounds(n, cap):
    """(first, last) rows of the chunks a group of n rows splits into when the grouped GEMMs
    tile it at most `cap` rows at a time: ceil(n / cap) chunks of equal size rounded up to
    16 rows, the last one ragged."""
    if n <= 0:
        return []
    nch = (n + cap - 1) // cap
    csz = ((n + nch - 1) // nch + 15) // 16 * 16
    return [(c * csz, min(n, (c + 1) * csz) - 1) for c in range(nch) if c * csz < n]


def chunk_covering_sample(idx, E, caps=(256, 128), hottest=8, n_min=256, seed=0):
    """Token sample for a full-size output check: the last row of every chunk (at every cap
    in `caps`) of the `hottest` experts, the first row of each of those experts, the last
    row of the last chunk of every expert split into more than one chunk, then random
    tokens up to n_min. Rows map to tokens through the stable permutation of `idx`.
    Returns (sorted distinct tokens, chunks covered)."""
    perm = oracle.permute(idx, E)
    offs, ptok = perm["offsets"], perm["perm_token"]
    counts = np.diff(offs[: E + 1])
    hot = np.argsort(-counts, kind="stable")[:hottest]
    toks, covered = set(), 0
    for e in range(E):
        for cap in caps:
            b = chunk_bounds(int(counts[e]), cap)
            if e in hot:
                toks.add(int(ptok[offs[e]]))
                for _, last in b:
                    toks.add(int(ptok[offs[e] + last]))
                covered += len(b)
            elif len(b) > 1:
                toks.add(int(ptok[offs[e] + b[-1][1]]))
                covered += 1
    rng = np.random.default_rng(seed)
    T = idx.shape[0]
    while len(toks) < min(n_min, T):
        toks.add(int(rng.integers(T)))
    return np.array(sorted(toks), np.int64), covered


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
