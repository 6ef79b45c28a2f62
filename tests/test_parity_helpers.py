"""Host checks of the parity helpers themselves (no GPU): the near-tie validator accepts a
valid tie-break and rejects a swap with an expert that is not tied, the chunk bounds follow
the grouped GEMMs' balanced split, and the covering sample reaches every chunk it names.

The "GPU answers" here are the oracle's own routing, edited on the CPU."""
import numpy as np
import pytest

import oracle
from _parity import check_near_ties, chunk_bounds, chunk_covering_sample, near_tie_tokens
from sparse_moe_layer_biased_b200.inputs import LayerShape, bf16_bits, draw


def _tied_case():
    # experts in identical pairs (same router row and bias), k odd: every token's k-th and
    # (k+1)-th experts are the two halves of one pair, margin exactly 0
    sh = LayerShape("ties", T=40, H=128, E=12, k=3, I=64, Is=64, seed=5)
    inp = draw(sh)
    inp["Wr"][1::2] = inp["Wr"][0::2]
    inp["bias"][1::2] = inp["bias"][0::2]
    o = oracle.router(bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].numpy(), sh.k, sh.scale, True)
    return sh, inp, o


def test_near_tie_validator_accepts_the_other_half_of_a_tied_pair():
    sh, inp, o = _tied_case()
    assert near_tie_tokens(o).size == sh.T
    assert check_near_ties(sh, inp, o["idx"], o["w"].astype(np.float32), o) == sh.T
    # take the other (higher-index) expert of the tied pair at rank k: still a valid top-k
    idx = o["idx"].copy()
    idx[:, sh.k - 1] += 1
    s = o["scores"]
    w = np.stack([sh.scale * s[t, idx[t]] / s[t, idx[t]].astype(np.float64).sum() for t in range(sh.T)])
    assert check_near_ties(sh, inp, idx, w.astype(np.float32), o) == sh.T


def test_near_tie_validator_rejects_an_expert_that_is_not_tied():
    sh, inp, o = _tied_case()
    b = o["scores"] + inp["bias"].numpy()[None, :]
    idx = o["idx"].copy()
    t = 0
    worst = int(np.argmin(b[t]))  # the lowest biased score: never within 1e-6 of the k-th
    idx[t, sh.k - 1] = worst
    with pytest.raises(AssertionError, match="not tied"):
        check_near_ties(sh, inp, idx, o["w"].astype(np.float32), o)


def test_near_tie_validator_rejects_wrong_weights():
    sh, inp, o = _tied_case()
    w = o["w"].astype(np.float32).copy()
    w[3, 0] *= 1.001
    with pytest.raises(AssertionError):
        check_near_ties(sh, inp, o["idx"], w, o)


@pytest.mark.parametrize("n,cap,expect", [
    (0, 256, []), (1, 256, [(0, 0)]), (256, 256, [(0, 255)]), (257, 256, [(0, 143), (144, 256)]),
    (300, 128, [(0, 111), (112, 223), (224, 299)]), (33, 32, [(0, 31), (32, 32)]),
])
def test_chunk_bounds(n, cap, expect):
    b = chunk_bounds(n, cap)
    assert b == expect
    if n:
        assert b[0][0] == 0 and b[-1][1] == n - 1
        assert all(b[i][1] + 1 == b[i + 1][0] for i in range(len(b) - 1))
        assert all(last - first + 1 <= cap for first, last in b)


def test_covering_sample_reaches_every_chunk_of_the_hot_experts():
    rng = np.random.default_rng(1)
    E, T, k = 20, 3000, 4
    p = np.r_[np.full(4, 0.15), np.full(16, 0.4 / 16)]
    idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    toks, covered = chunk_covering_sample(idx, E, caps=(256, 128), hottest=4, n_min=50)
    perm = oracle.permute(idx, E)
    offs, slot_of = perm["offsets"], perm["slot_of"]
    counts = np.diff(offs[:E + 1])
    hot = np.argsort(-counts, kind="stable")[:4]
    rows_hit = set(int(slot_of[t, j]) for t in toks for j in range(k))
    for e in hot:
        for cap in (256, 128):
            for first, last in chunk_bounds(int(counts[e]), cap):
                assert any(offs[e] + first <= r <= offs[e] + last for r in rows_hit)
    assert len(toks) >= 50 and covered > 0
