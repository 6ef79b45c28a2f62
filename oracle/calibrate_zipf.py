"""Calibrate gamma of the skewed workload's Zipf-shaped router bias with the CPU oracle.

The skewed Step-5-Preview workload asks for expert load following Zipf(s = 1.1)
over a random expert permutation, with the hottest 8 experts taking about 30% of
the assignments. The bias is bias[perm[r]] = -gamma * s * ln(r + 1); this script
finds gamma by bisection (40 fixed iterations, fp64 on the host) so that the
oracle router, run on tokens drawn like that workload, gives a hottest-8 share of
0.30. With --write it stores the result as ZIPF_GAMMA in the input module.

Run: python -m oracle.calibrate_zipf [--tokens 4096] [--write]
"""
from __future__ import annotations

import argparse
import os
import re
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

import oracle  # noqa: E402
from sparse_moe_layer_biased_b200 import inputs  # noqa: E402


def hottest8_share(logits, bias, k):
    sel = oracle.router_select(logits, bias, k)
    counts = np.bincount(sel["idx"].ravel(), minlength=logits.shape[1])
    top = np.sort(counts)[::-1]
    return float(top[:8].sum()) / float(counts.sum()), top


def calibrate(tokens: int, target: float = 0.30, iters: int = 40):
    shape = inputs.WORKLOADS["step5_skewed"].replace(T=tokens)
    r = inputs.draw_router_only(shape, gamma=0.0)
    logits = oracle.router_logits(inputs.bf16_bits(r["x"]), inputs.bf16_bits(r["Wr"]))
    lo, hi = 0.0, 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        bias = inputs.zipf_bias(shape.E, shape.seed, mid).numpy()
        share, _ = hottest8_share(logits, bias, shape.k)
        if share < target:
            lo = mid
        else:
            hi = mid
    gamma = 0.5 * (lo + hi)
    share, top = hottest8_share(logits, inputs.zipf_bias(shape.E, shape.seed, gamma).numpy(), shape.k)
    return gamma, share, top


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--write", action="store_true")
    a = ap.parse_args()
    gamma, share, top = calibrate(a.tokens)
    tot = top.sum()
    print(f"gamma={gamma:.6f} hottest8_share={share:.4f} top1_share={top[0] / tot:.4f} "
          f"empty_experts={(top == 0).sum()}")
    if a.write:
        path = os.path.join(os.path.dirname(HERE), "sparse_moe_layer_biased_b200", "inputs.py")
        src = open(path).read()
        src = re.sub(r"^ZIPF_GAMMA = .*$", f"ZIPF_GAMMA = {gamma:.6f}", src, flags=re.M)
        open(path, "w").write(src)
        print("wrote", path)


if __name__ == "__main__":
    main()
