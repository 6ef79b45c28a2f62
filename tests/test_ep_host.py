"""Expert-parallel exchange (sparse_moe_layer_biased_b200.ep) as gloo ranks on the CPU.

The product layer runs every arithmetic step in the CUDA library; what crosses ranks is the
data movement of ep.dispatch / ep.combine_back and the layout contract between them: slots
in global expert order go out owner-major, rows arrive source-major and expert-minor, and
the outputs come back to the slots they left. Here the ranks route with the oracle, pack
in the slot order of moe_permute's contract (the oracle's permutation), exchange through
the product helpers, compute the received rows with the oracle's expert MLP, and must
reproduce, on every rank, the oracle's whole-layer output for that rank's tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_moe_layer_biased_b200.inputs import LayerShape, bf16_bits, draw

SHAPE = LayerShape("ep_host", T=8, H=64, E=8, k=3, I=64, Is=64, limit_routed=0.25, limit_shared=0.125, seed=61,
                   weight_std=0.05)
TOKENS = [29, 18, 0, 11]  # tokens per rank (rank 2 has none)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _bf16_tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _rank_step(rank, world):
    import oracle
    from sparse_moe_layer_biased_b200 import ep

    sh = SHAPE
    W = draw(sh)  # common weights: every rank draws the same
    Wr, bias = bf16_bits(W["Wr"]), W["bias"].numpy()
    gu, dn = bf16_bits(W["W_gate_up"]), bf16_bits(W["W_down"])
    shg, shd = bf16_bits(W["Wsh_gate_up"]), bf16_bits(W["Wsh_down"])
    T = TOKENS[rank]
    x = bf16_bits(draw(sh.replace(T=max(T, 1), seed=100 + rank))["x"])[:T]
    Er = sh.E // world
    k, H = sh.k, sh.H

    # route and permute (the oracle's forms of moe_router and moe_permute)
    if T > 0:
        r = oracle.router(x, Wr, bias, k, sh.scale, sh.norm_expert_weight)
        p = oracle.permute(r["idx"], sh.E)
        w = r["w"]
    else:
        p = {"counts": np.zeros(sh.E + 1, np.int32), "perm_token": np.zeros(0, np.int32),
             "slot_of": np.zeros((0, k), np.int32)}
        w = np.zeros((0, k))
    # pack: the contract of moe_ep_pack
    x_send = np.zeros((T * k, H), np.uint16)
    w_send = np.zeros((T * k,), np.float64)
    for t in range(T):
        for j in range(k):
            s = p["slot_of"][t, j]
            x_send[s] = x[t]
            w_send[s] = w[t, j]
    send_ce = ep.ep_counts(torch.from_numpy(p["counts"].astype(np.int32)), world)
    x_recv, w_recv, recv_ce, send_rows, recv_rows = ep.dispatch(_bf16_tensor(x_send), torch.from_numpy(w_send),
                                                                send_ce)
    assert list(recv_ce.sum(1)) == recv_rows and sum(send_rows) == T * k

    # owner side: rows source-major, expert-minor (the contract of moe_ep_experts)
    xr = x_recv.view(torch.int16).numpy().view(np.uint16)
    out_recv = np.zeros((xr.shape[0], H), np.float64)
    n = 0
    for s in range(world):
        for e in range(Er):
            g = rank * Er + e
            for _ in range(int(recv_ce[s, e])):
                out_recv[n] = float(w_recv[n]) * oracle.swiglu_mlp(xr[n], gu[g], dn[g], sh.limit_routed)
                n += 1
    assert n == xr.shape[0]

    o_slots = torch.zeros((T * k, H), dtype=torch.float64)
    ep.combine_back(torch.from_numpy(out_recv), o_slots, send_rows, recv_rows)
    o = o_slots.numpy()
    y = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            y[t] += o[p["slot_of"][t, j]]
        y[t] += oracle.swiglu_mlp(x[t], shg, shd, sh.limit_shared)
    if T > 0:
        experts = {e: (gu[e], dn[e]) for e in range(sh.E)}
        ref = oracle.forward_tokens(x, Wr, bias, experts, shg, shd, k=k, scale=sh.scale,
                                    norm=sh.norm_expert_weight, limit_routed=sh.limit_routed,
                                    limit_shared=sh.limit_shared)["y"]
        np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)
    return T, int(sum(recv_rows))


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = _rank_step(rank, world)
    except Exception as e:  # reported by the parent
        out[rank] = repr(e)
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_exchange_reproduces_the_layer(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        assert isinstance(res[rank], tuple), res[rank]
    # every routed (token, rank) entry was computed exactly once somewhere
    assert sum(r[1] for r in res.values()) == sum(TOKENS[:world]) * SHAPE.k


def test_ep_counts_splits_owner_major():
    from sparse_moe_layer_biased_b200 import ep

    counts = torch.arange(9, dtype=torch.int32)  # E = 8 experts + shared
    ce = ep.ep_counts(counts, 4)
    assert ce.tolist() == [[0, 1], [2, 3], [4, 5], [6, 7]]
    with pytest.raises(ValueError):
        ep.ep_counts(counts, 3)
