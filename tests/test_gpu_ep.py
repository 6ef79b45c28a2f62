"""GPU parity of the expert-parallel pieces (moe_ep_pack, moe_ep_experts, moe_shared_expert,
EPMoeLayer) against the oracle.

One GPU is available, so the owner side (moe_ep_experts) is driven with synthetic receive
layouts from several sources, which is a local computation, and the whole layer runs on a
one-rank NCCL group (the all-to-alls are then copies). Cross-rank data movement is covered
by tests/test_ep_host.py with gloo ranks. Tolerances as in the layer's parity tests.
"""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from _parity import check_output, check_routing, oracle_router, rel_fro
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.ep import EPMoeLayer
from sparse_moe_layer_biased_b200.inputs import LayerShape, bf16_bits, draw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    _abi.lib()
    yield
    _abi.moe_check_device()


def _local_desc(sh, rows, Er):
    return _abi.LayerDesc(rows, sh.H, Er, 1, sh.I, sh.Is, sh.scale, int(sh.norm_expert_weight), sh.limit_routed,
                          sh.limit_shared, 0)


# (shape, per-source row counts [R, Er]): sizes span several 128-row tiles with ragged tails,
# empty experts and an empty source; the second runs on CTA pairs (H % 512, I % 128).
CASES = {
    "three_sources": (LayerShape("ep_own", T=1, H=512, E=5, k=1, I=192, Is=128, limit_routed=0.25, seed=71,
                                 weight_std=0.03),
                      [[40, 0, 133, 7, 90], [0, 0, 0, 0, 0], [61, 150, 2, 0, 35]]),
    "pairs": (LayerShape("ep_own_pair", T=1, H=1024, E=4, k=1, I=256, Is=256, limit_routed=0.0, seed=72,
                         weight_std=0.03),
              [[300, 5, 0, 260], [17, 280, 64, 1]]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_ep_experts_against_oracle(name):
    sh, counts = CASES[name]
    R, Er = len(counts), sh.E
    ce = np.asarray(counts, np.int32)
    n = int(ce.sum())
    W = draw(sh)
    g = torch.Generator().manual_seed(sh.seed)
    x_recv = (torch.randn((n, sh.H), generator=g) * 1.0).to(torch.bfloat16)
    w_recv = torch.rand((n,), generator=g) * 0.9 + 0.1
    dev = {"x": x_recv.cuda(), "w": w_recv.cuda(), "ce": torch.from_numpy(ce).cuda(),
           "gu": W["W_gate_up"].cuda(), "d": W["W_down"].cuda()}
    dl = _local_desc(sh, n, Er)
    ws = torch.empty(_abi.moe_workspace_size(dl), dtype=torch.uint8, device="cuda")
    out = torch.full((n, sh.H), float("nan"), dtype=torch.float32, device="cuda")
    _abi.moe_ep_experts(dl, R, dev["ce"], dev["x"], dev["w"], dev["gu"], dev["d"], out, ws)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    got = out.cpu().numpy()
    xb, gu, dn = bf16_bits(x_recv), bf16_bits(W["W_gate_up"]), bf16_bits(W["W_down"])
    ref = np.zeros((n, sh.H))
    r = 0
    for s in range(R):
        for e in range(Er):
            for _ in range(int(ce[s, e])):
                ref[r] = float(w_recv[r]) * oracle.swiglu_mlp(xb[r], gu[e], dn[e], sh.limit_routed)
                r += 1
    assert np.isfinite(got).all()
    rf, ma = check_output(got, ref, name)
    print(f"{name}: rows {n} rel_fro {rf:.2e} max_abs {ma:.2e}")


def test_ep_experts_nothing_received():
    sh, _ = CASES["three_sources"]
    dl = _local_desc(sh, 0, sh.E)
    _abi.moe_ep_experts(dl, 3, None, None, None, None, None, None, None)


def test_shared_expert_against_oracle():
    sh = LayerShape("ep_shared", T=333, H=512, E=6, k=2, I=128, Is=192, limit_shared=0.125, seed=73, weight_std=0.03)
    W = draw(sh)
    dev = {k: v.cuda() for k, v in W.items()}
    d = _abi.desc_of(sh)
    ws = torch.empty(_abi.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    out = torch.full((sh.T, sh.H), float("nan"), dtype=torch.float32, device="cuda")
    _abi.moe_shared_expert(d, dev["x"], dev["Wsh_gate_up"], dev["Wsh_down"], out, ws)
    torch.cuda.synchronize()
    xb, shg, shd = bf16_bits(W["x"]), bf16_bits(W["Wsh_gate_up"]), bf16_bits(W["Wsh_down"])
    ref = np.stack([oracle.swiglu_mlp(xb[t], shg, shd, sh.limit_shared) for t in range(sh.T)])
    check_output(out.cpu().numpy(), ref, "shared")


def test_ep_pack_rows_and_weights():
    sh = LayerShape("ep_pack", T=77, H=256, E=8, k=3, I=64, Is=64, seed=74)
    W = {k: v.cuda() for k, v in draw(sh).items()}
    d = _abi.desc_of(sh)
    T, k = sh.T, sh.k
    g = torch.Generator().manual_seed(3)
    idx = torch.stack([torch.randperm(sh.E, generator=g)[:k] for _ in range(T)]).to(torch.int32).cuda()
    w = torch.rand((T, k), generator=g).cuda()
    counts = torch.empty(sh.E + 1, dtype=torch.int32, device="cuda")
    offsets = torch.empty(sh.E + 2, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k + T, dtype=torch.int32, device="cuda")
    slot_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
    _abi.moe_permute(d, idx, counts, offsets, perm, slot_of)
    x_send = torch.empty((T * k, sh.H), dtype=torch.bfloat16, device="cuda")
    w_send = torch.empty((T * k,), dtype=torch.float32, device="cuda")
    _abi.moe_ep_pack(d, W["x"], w, slot_of, x_send, w_send)
    torch.cuda.synchronize()
    so = slot_of.cpu().numpy()
    tok = np.repeat(np.arange(T), k)
    assert np.array_equal(bf16_bits(x_send)[so.ravel()], bf16_bits(W["x"])[tok])
    assert np.array_equal(w_send.cpu().numpy()[so.ravel()], w.cpu().numpy().ravel())
    # owner-major: the slots of experts [r*Er, (r+1)*Er) are contiguous and in that order
    p = oracle.permute(idx.cpu().numpy(), sh.E)
    assert np.array_equal(so, p["slot_of"])


@pytest.fixture(scope="module")
def one_rank_group(tmp_path_factory):
    store = dist.FileStore(str(tmp_path_factory.mktemp("ep") / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


EP_SHAPES = {
    "ep_layer": LayerShape("ep_layer", T=300, H=512, E=12, k=4, I=256, Is=256, limit_routed=0.25,
                           limit_shared=0.125, seed=75),
    "ep_layer_ragged": LayerShape("ep_layer_ragged", T=173, H=384, E=10, k=3, I=192, Is=128, seed=76),
}


@pytest.mark.parametrize("name", list(EP_SHAPES))
def test_ep_layer_one_rank_against_oracle(one_rank_group, name):
    sh = EP_SHAPES[name]
    inp = draw(sh)
    dev = {k: v.cuda() for k, v in inp.items()}
    layer = EPMoeLayer(sh, dev, group=one_rank_group)
    y, idx, w = layer.forward(dev["x"], routing=True)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    ref = oracle.forward_full(inp, sh)
    keep = check_routing(idx.cpu().numpy(), w.cpu().numpy(), ref, sh.E, sh.k)
    check_output(y.cpu().numpy()[keep], ref["y"][keep], name)
    # the combine sums in a fixed order: two calls agree bit for bit
    y2 = layer.forward(dev["x"])
    assert torch.equal(y, y2)
    # and the single-GPU layer agrees to rounding
    from sparse_moe_layer_biased_b200.layer import MoeLayer
    y1 = MoeLayer(sh, dev).forward(dev["x"])
    assert rel_fro(y.cpu().numpy(), y1.cpu().numpy()) < 1e-5


def test_ep_layer_zero_tokens(one_rank_group):
    sh = EP_SHAPES["ep_layer"]
    dev = {k: v.cuda() for k, v in draw(sh).items()}
    layer = EPMoeLayer(sh, dev, group=one_rank_group)
    y = layer.forward(dev["x"][:0])
    torch.cuda.synchronize()
    assert y.shape == (0, sh.H)
