"""Bounded device waits, exercised without faulting the GPU.

Every mbarrier wait in the kernels gives up after the wait limit (moe_set_wait_limit_ns),
sets the library's device error word and lets the CTA drain its own copies and MMAs,
free its TMEM and return. With a 1 us limit, waits for data from HBM run out (L2 is
flushed first); the test checks that moe_check_device then reports MOE_ERR_TIMEOUT and
that, with the default limit restored, the same layer runs again and matches the oracle.
No kernel traps, faults or waits without a bound.
"""
import numpy as np
import pytest
import torch

import oracle
from _parity import check_output, check_routing
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import WORKLOADS, LayerShape, draw
from sparse_moe_layer_biased_b200.layer import MoeLayer

pytestmark = pytest.mark.gpu

SHAPES = {
    "decode_config": WORKLOADS["tiny"],
    "single_cta": LayerShape("mt2", T=300, H=768, E=12, k=4, I=256, Is=128, limit_routed=0.25, seed=27,
                             weight_std=0.03),
    "cta_pairs": LayerShape("pair", T=300, H=512, E=12, k=4, I=256, Is=256, limit_routed=0.25, seed=29,
                            weight_std=0.03),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_short_wait_limit_reports_timeout_and_recovers(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    sh = SHAPES[name]
    inp_h = draw(sh)
    inp = {k: v.cuda() for k, v in inp_h.items()}
    layer = MoeLayer(sh, inp)
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")  # 256 MB > L2
    _abi.moe_check_device()
    statuses = []
    old = _abi.moe_set_wait_limit_ns(1000)
    try:
        for _ in range(4):
            flush.fill_(1.0)
            layer.forward(inp["x"])
            try:
                _abi.moe_check_device()
                statuses.append("ok")
            except _abi.MoeError as e:
                assert e.status == 5, e
                statuses.append("timeout")
    finally:
        _abi.moe_set_wait_limit_ns(old)
    assert "timeout" in statuses, statuses
    # the context is still usable and the layer is right again
    y, idx, w = layer.forward(inp["x"], routing=True)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    ref = oracle.forward_full(inp_h, sh)
    keep = check_routing(idx.cpu().numpy(), w.cpu().numpy(),
                         {"idx": ref["idx"], "w": ref["w"], "margin": ref["margin"]}, sh.E, sh.k)
    check_output(y.cpu().numpy()[keep], ref["y"][keep], name)
