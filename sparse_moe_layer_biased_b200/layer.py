"""MoeLayer: device-resident weights + workspace around the moe_forward entry point.

PyTorch only allocates device memory and supplies the stream; the layer's arithmetic
runs in libmoe_b200.so.
"""
from __future__ import annotations

import torch

from . import _abi


class MoeLayer:
    """One MoE layer call shape (inputs.LayerShape) with its weights on a CUDA device.

    weights: dict with Wr [E, H] bf16, bias [E] fp32, W_gate_up [E, 2I, H] bf16,
    W_down [E, H, I] bf16, Wsh_gate_up [2Is, H] bf16, Wsh_down [H, Is] bf16. With FP8 E4M3
    routed experts the dict holds W_gate_up_q [E, 2I, H] / W_down_q [E, H, I] uint8 codes
    and their 128x128 block scales W_gate_up_s / W_down_s (fp32) instead of W_gate_up /
    W_down, and forward runs moe_forward_fp8.
    """

    def __init__(self, shape, weights: dict, deterministic: bool = False, max_tokens: int | None = None):
        self.shape = shape
        self.deterministic = deterministic
        self.w = weights
        self.fp8 = "W_gate_up_q" in weights
        dev = weights["Wr"].device
        self.max_tokens = shape.T if max_tokens is None else max_tokens
        nbytes = _abi.moe_workspace_size(_abi.desc_of(shape, T=self.max_tokens, deterministic=deterministic))
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, routing: bool = False, stream=None):
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"{T} tokens exceed the workspace size of {self.max_tokens}")
        desc = _abi.desc_of(self.shape, T=T, deterministic=self.deterministic)
        if y is None:
            y = torch.empty((T, self.shape.H), dtype=torch.float32, device=x.device)
        idx = w = None
        if routing:
            idx = torch.empty((T, self.shape.k), dtype=torch.int32, device=x.device)
            w = torch.empty((T, self.shape.k), dtype=torch.float32, device=x.device)
        W = self.w
        if self.fp8:
            _abi.moe_forward_fp8(desc, x, W["Wr"], W["bias"], W["W_gate_up_q"], W["W_gate_up_s"], W["W_down_q"],
                                 W["W_down_s"], W["Wsh_gate_up"], W["Wsh_down"], y, self.ws, idx, w, stream=stream)
        else:
            _abi.moe_forward(desc, x, W["Wr"], W["bias"], W["W_gate_up"], W["W_down"], W["Wsh_gate_up"],
                             W["Wsh_down"], y, self.ws, idx, w, stream=stream)
        return (y, idx, w) if routing else y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor | None = None, stream=None):
        """The layer over batches in host memory: x_host [n, T, H] bf16 -> y_host [n, T, H]
        fp32 (page-locked tensors for overlapped copies) through moe_forward_host, with BF16
        or FP8 routed experts. Returns y_host once the work is enqueued; synchronize the
        stream before reading it."""
        n, T, H = x_host.shape
        if T > self.max_tokens:
            raise ValueError(f"{T} tokens exceed the workspace size of {self.max_tokens}")
        desc = _abi.desc_of(self.shape, T=T, deterministic=self.deterministic)
        need = _abi.moe_host_workspace_size(desc)
        if getattr(self, "ws_host", None) is None or self.ws_host.numel() < need:
            self.ws_host = torch.empty(need, dtype=torch.uint8, device=self.w["Wr"].device)
        if y_host is None:
            y_host = torch.empty((n, T, H), dtype=torch.float32, pin_memory=True)
        W = self.w
        if self.fp8:
            _abi.moe_forward_host(desc, n, x_host, W["Wr"], W["bias"], W["W_gate_up_q"], W["W_down_q"],
                                  W["Wsh_gate_up"], W["Wsh_down"], y_host, self.ws_host, stream=stream,
                                  W_gate_up_scale=W["W_gate_up_s"], W_down_scale=W["W_down_s"])
        else:
            _abi.moe_forward_host(desc, n, x_host, W["Wr"], W["bias"], W["W_gate_up"], W["W_down"],
                                  W["Wsh_gate_up"], W["Wsh_down"], y_host, self.ws_host, stream=stream)
        return y_host
