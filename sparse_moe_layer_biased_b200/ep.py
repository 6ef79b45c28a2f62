"""Expert-parallel (DP_EP) form of the layer over a torch.distributed process group.

"MAX 中 Step-3.5-Flash 架构解析", section "并行模式TP_TP / TP_EP / DP_EP": in DP_EP every rank
runs its own batch shard, the routed experts are split across the ranks and an EP combine
follows the MoE (the NeMo AutoModel Step-5-Preview page lists expert parallelism, e.g. EP32
with 11 routed experts per rank). Rank r of R owns the routed experts [r*Er, (r+1)*Er),
Er = E / R; the router weights, the router bias and the shared expert are replicated.

One forward on each rank (one process per GPU):
  1. moe_router and moe_permute over the global E experts: routed slots in global expert
     order, which is (owner rank, local expert) order;
  2. moe_ep_pack: the send rows x_send[slot] = x[token] and their routing weights;
  3. moe_shared_expert writes rows [T*k, T*k + T) of o_perm: it needs no routing, so it is
     enqueued before the host waits for the counts below and keeps the GPU busy meanwhile;
  4. dispatch: an all-to-all of the [R, Er] per-(owner, local expert) row counts, then of the
     rows and weights, which arrive source-major (source 0's rows for its local expert 0, 1,
     ..., then source 1's);
  5. moe_ep_experts: this rank's experts on the received rows, one weighted fp32 output row
     per received row, in received order;
  6. return: the reverse all-to-all puts every output row back at its slot, rows [0, T*k)
     of o_perm;
  7. moe_combine: y[t] = sum over j of o_perm[slot_of[t, j]] + o_perm[T*k + t], in a fixed
     order, so the result does not depend on R.

The all-to-alls are NCCL collectives issued through torch.distributed (plumbing); every
arithmetic step runs in libmoe_b200.so. The counts are read on the host once per forward
to size the row exchange (torch.distributed's all-to-all takes host split sizes), after
the shared expert has been enqueued. Only routed BF16 experts are supported here.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _abi


def ep_counts(counts: torch.Tensor, ranks: int) -> torch.Tensor:
    """[R, Er] rows per (owner rank, local expert) from moe_permute's counts [E + 1]."""
    E = counts.numel() - 1
    if E % ranks:
        raise ValueError(f"{E} experts do not split over {ranks} ranks")
    return counts[:E].view(ranks, E // ranks).contiguous()


def dispatch(x_send: torch.Tensor, w_send: torch.Tensor, send_ce: torch.Tensor, group=None):
    """Rows of x_send / w_send (slot order, owner-major) to their owners.

    Returns (x_recv, w_recv, recv_ce, send_rows, recv_rows): recv_ce [R, Er] holds the rows
    each source sent for each local expert, send_rows / recv_rows the per-rank row counts
    (host lists) that the return exchange reuses."""
    recv_ce = torch.empty_like(send_ce)
    dist.all_to_all_single(recv_ce, send_ce, group=group)
    send_rows = send_ce.sum(1).tolist()
    recv_rows = recv_ce.sum(1).tolist()
    n = int(sum(recv_rows))
    x_recv = torch.empty((n, x_send.shape[1]), dtype=x_send.dtype, device=x_send.device)
    w_recv = torch.empty((n,), dtype=w_send.dtype, device=w_send.device)
    dist.all_to_all_single(x_recv, x_send, recv_rows, send_rows, group=group)
    dist.all_to_all_single(w_recv, w_send, recv_rows, send_rows, group=group)
    return x_recv, w_recv, recv_ce, send_rows, recv_rows


def combine_back(out_recv: torch.Tensor, out_slots: torch.Tensor, send_rows, recv_rows, group=None):
    """Output rows computed by the owners back to the slots they came from: out_slots
    [sum(send_rows), H] receives them in the order the rows were sent."""
    dist.all_to_all_single(out_slots, out_recv, send_rows, recv_rows, group=group)
    return out_slots


class EPMoeLayer:
    """The layer with its routed experts split over the ranks of `group`.

    weights: Wr [E, H] bf16, bias [E] fp32, Wsh_gate_up [2Is, H] bf16, Wsh_down [H, Is] bf16
    (replicated) and this rank's experts W_gate_up [Er, 2I, H], W_down [Er, H, I] bf16."""

    def __init__(self, shape, weights: dict, group=None, max_tokens: int | None = None):
        self.shape = shape
        self.group = group
        self.R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if shape.E % self.R:
            raise ValueError(f"{shape.E} experts do not split over {self.R} ranks")
        self.Er = shape.E // self.R
        if weights["W_gate_up"].shape[0] != self.Er or weights["W_down"].shape[0] != self.Er:
            raise ValueError(f"rank {self.rank} must hold {self.Er} routed experts")
        self.w = weights
        dev = weights["Wr"].device
        self.max_tokens = shape.T if max_tokens is None else max_tokens
        nbytes = _abi.moe_workspace_size(_abi.desc_of(shape, T=self.max_tokens))
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.ws_experts = torch.empty(0, dtype=torch.uint8, device=dev)

    def _local_desc(self, rows: int) -> _abi.LayerDesc:
        sh = self.shape
        return _abi.LayerDesc(rows, sh.H, self.Er, 1, sh.I, sh.Is, sh.scale, int(bool(sh.norm_expert_weight)),
                              sh.limit_routed, sh.limit_shared, 0)

    def forward(self, x: torch.Tensor, routing: bool = False):
        sh, W, dev = self.shape, self.w, x.device
        T, k, H, E = x.shape[0], sh.k, sh.H, sh.E
        if T > self.max_tokens:
            raise ValueError(f"{T} tokens exceed the workspace size of {self.max_tokens}")
        d = _abi.desc_of(sh, T=T)
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        counts = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        offsets = torch.empty((E + 2,), dtype=torch.int32, device=dev)
        perm_token = torch.empty((T * k + T,), dtype=torch.int32, device=dev)
        slot_of = torch.empty((T, k), dtype=torch.int32, device=dev)
        x_send = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
        w_send = torch.empty((T * k,), dtype=torch.float32, device=dev)
        o_perm = torch.empty((T * k + T, H), dtype=torch.float32, device=dev)
        if T > 0:
            _abi.moe_router(d, x, W["Wr"], W["bias"], idx, w)
            _abi.moe_permute(d, idx, counts, offsets, perm_token, slot_of)
            _abi.moe_ep_pack(d, x, w, slot_of, x_send, w_send)
            _abi.moe_shared_expert(d, x, W["Wsh_gate_up"], W["Wsh_down"], o_perm[T * k:], self.ws)
        else:
            counts.zero_()
        x_recv, w_recv, recv_ce, send_rows, recv_rows = dispatch(x_send, w_send, ep_counts(counts, self.R),
                                                                  self.group)
        n = x_recv.shape[0]
        dl = self._local_desc(n)
        need = _abi.moe_workspace_size(dl)
        if self.ws_experts.numel() < need:
            self.ws_experts = torch.empty(need, dtype=torch.uint8, device=dev)
        out_recv = torch.empty((n, H), dtype=torch.float32, device=dev)
        _abi.moe_ep_experts(dl, self.R, recv_ce, x_recv, w_recv, W["W_gate_up"], W["W_down"], out_recv,
                            self.ws_experts)
        combine_back(out_recv, o_perm[: T * k], send_rows, recv_rows, self.group)
        y = torch.empty((T, H), dtype=torch.float32, device=dev)
        if T > 0:
            _abi.moe_combine(d, o_perm, slot_of, y)
        return (y, idx, w) if routing else y
