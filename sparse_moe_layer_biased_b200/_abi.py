"""ctypes binding of libmoe_b200.so: argument marshalling only.

Every function here takes torch tensors (or None), passes their device pointers and
sizes to the C entry point of the same name, and raises MoeError on a non-zero
status. All computation happens in the library's CUDA kernels; there is no fallback:
if the library is missing this module raises on import of the first call.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_B200_DEBUG=1 loads the debug build (device-side range checks, MOE_ERR_DEVICE_BOUNDS)
DEBUG = os.environ.get("MOE_B200_DEBUG", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libmoe_b200_debug.so" if DEBUG else "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_BOUNDS"}

# Every exported entry point; the header include/moe_b200.h declares exactly these.
EXPORTS = ["moe_status_string", "moe_workspace_size", "moe_router", "moe_permute", "moe_expert_ffn",
           "moe_combine", "moe_forward", "moe_check_device", "moe_set_wait_limit_ns", "moe_set_stage_events",
           "moe_forward_noalloc", "moe_forward_with_ids", "moe_forward_fp8", "moe_backward",
           "moe_backward_workspace_size", "moe_ep_pack", "moe_ep_experts", "moe_shared_expert",
           "moe_host_workspace_size", "moe_forward_host"]


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


class LayerDesc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("Is", ctypes.c_int32), ("scale", ctypes.c_float),
                ("norm_expert_weight", ctypes.c_int32), ("limit_routed", ctypes.c_float),
                ("limit_shared", ctypes.c_float), ("deterministic", ctypes.c_int32)]


def desc_of(shape, T=None, deterministic=False) -> LayerDesc:
    """LayerDesc from an inputs.LayerShape (T overridable)."""
    return LayerDesc(shape.T if T is None else T, shape.H, shape.E, shape.k, shape.I, shape.Is, shape.scale,
                     int(bool(shape.norm_expert_weight)), shape.limit_routed, shape.limit_shared,
                     int(bool(deterministic)))


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run __graft_entry__.build() or "
                               "python -m sparse_moe_layer_biased_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        dp = ctypes.POINTER(LayerDesc)
        L.moe_status_string.argtypes = [i32]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
        L.moe_router.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp]
        L.moe_permute.argtypes = [dp, vp, vp, vp, vp, vp, vp]
        L.moe_expert_ffn.argtypes = [dp] + [vp] * 11 + [sz, vp]
        L.moe_combine.argtypes = [dp, vp, vp, vp, vp]
        L.moe_forward.argtypes = [dp] + [vp] * 11 + [sz, vp]
        L.moe_check_device.argtypes = []
        L.moe_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.moe_set_wait_limit_ns.restype = ctypes.c_uint64
        L.moe_set_stage_events.argtypes = [ctypes.POINTER(vp), i32]
        L.moe_forward_with_ids.argtypes = [dp] + [vp] * 9 + [sz, vp]
        L.moe_forward_fp8.argtypes = [dp] + [vp] * 13 + [sz, vp]
        L.moe_backward_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
        L.moe_backward.argtypes = [dp] + [vp] * 16 + [sz, vp]
        L.moe_forward_with_ids.restype = i32
        L.moe_forward_noalloc.argtypes = [dp] + [vp] * 11
        L.moe_forward_noalloc.restype = i32
        L.moe_ep_pack.argtypes = [dp] + [vp] * 6
        L.moe_ep_experts.argtypes = [dp, ctypes.c_int32] + [vp] * 7 + [sz, vp]
        L.moe_shared_expert.argtypes = [dp] + [vp] * 5 + [sz, vp]
        L.moe_host_workspace_size.argtypes = [dp, ctypes.POINTER(sz)]
        L.moe_forward_host.argtypes = [dp, ctypes.c_int32] + [vp] * 11 + [sz, vp]
        for name in ("moe_ep_pack", "moe_ep_experts", "moe_shared_expert", "moe_host_workspace_size",
                     "moe_forward_host"):
            getattr(L, name).restype = i32
        for name in ("moe_workspace_size", "moe_router", "moe_permute", "moe_expert_ffn", "moe_combine",
                     "moe_forward", "moe_check_device", "moe_set_stage_events"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, st):
    if st != MOE_OK:
        raise MoeError(fn, st)


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_workspace_size(desc: LayerDesc) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(desc), ctypes.byref(out)))
    return out.value


def moe_router(desc, x, Wr, bias, topk_idx, topk_w, margin=None, stream=None):
    _check("moe_router", lib().moe_router(ctypes.byref(desc), _p(x), _p(Wr), _p(bias), _p(topk_idx), _p(topk_w),
                                          _p(margin), _stream(stream)))


def moe_permute(desc, topk_idx, counts, offsets, perm_token, slot_of, stream=None):
    _check("moe_permute", lib().moe_permute(ctypes.byref(desc), _p(topk_idx), _p(counts), _p(offsets),
                                            _p(perm_token), _p(slot_of), _stream(stream)))


def moe_expert_ffn(desc, x, topk_w, offsets, perm_token, slot_of, W_gate_up, W_down, Wsh_gate_up, Wsh_down, out,
                   ws, stream=None):
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        ctypes.byref(desc), _p(x), _p(topk_w), _p(offsets), _p(perm_token), _p(slot_of), _p(W_gate_up),
        _p(W_down), _p(Wsh_gate_up), _p(Wsh_down), _p(out), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_combine(desc, o_perm, slot_of, y, stream=None):
    _check("moe_combine", lib().moe_combine(ctypes.byref(desc), _p(o_perm), _p(slot_of), _p(y), _stream(stream)))


def moe_forward(desc, x, Wr, bias, W_gate_up, W_down, Wsh_gate_up, Wsh_down, y, ws, topk_idx_out=None,
                topk_w_out=None, stream=None):
    _check("moe_forward", lib().moe_forward(
        ctypes.byref(desc), _p(x), _p(Wr), _p(bias), _p(W_gate_up), _p(W_down), _p(Wsh_gate_up), _p(Wsh_down),
        _p(y), _p(topk_idx_out), _p(topk_w_out), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_forward_fp8(desc, x, Wr, bias, W_gate_up_q, W_gate_up_scale, W_down_q, W_down_scale, Wsh_gate_up,
                    Wsh_down, y, ws, topk_idx_out=None, topk_w_out=None, stream=None):
    """The layer with FP8 E4M3 routed experts (uint8 codes + fp32 128x128 block scales)."""
    _check("moe_forward_fp8", lib().moe_forward_fp8(
        ctypes.byref(desc), _p(x), _p(Wr), _p(bias), _p(W_gate_up_q), _p(W_gate_up_scale), _p(W_down_q),
        _p(W_down_scale), _p(Wsh_gate_up), _p(Wsh_down), _p(y), _p(topk_idx_out), _p(topk_w_out), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_backward_workspace_size(desc) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_backward_workspace_size", lib().moe_backward_workspace_size(ctypes.byref(desc), ctypes.byref(out)))
    return int(out.value)


def moe_backward(desc, x, Wr, W_gate_up, W_down, Wsh_gate_up, Wsh_down, topk_idx, topk_w, dy, dx, dWr, dW_gate_up,
                 dW_down, dWsh_gate_up, dWsh_down, ws, stream=None):
    """Gradients of the layer for the forward's routing and dy (all outputs overwritten)."""
    _check("moe_backward", lib().moe_backward(
        ctypes.byref(desc), _p(x), _p(Wr), _p(W_gate_up), _p(W_down), _p(Wsh_gate_up), _p(Wsh_down), _p(topk_idx),
        _p(topk_w), _p(dy), _p(dx), _p(dWr), _p(dW_gate_up), _p(dW_down), _p(dWsh_gate_up), _p(dWsh_down), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))


def moe_check_device():
    _check("moe_check_device", lib().moe_check_device())


def moe_set_wait_limit_ns(ns: int) -> int:
    return int(lib().moe_set_wait_limit_ns(ns))


def moe_set_stage_events(events) -> None:
    """events: list of torch.cuda.Event (enable_timing=True), or [] to turn the hook off.

    torch creates an event's CUDA handle on its first record, so events without a handle
    are recorded once here on the current stream to materialise it.
    """
    for ev in events:
        if not ev.cuda_event:
            ev.record()
    n = len(events)
    arr = (ctypes.c_void_p * max(n, 1))(*[ev.cuda_event for ev in events])
    _check("moe_set_stage_events", lib().moe_set_stage_events(arr if n else None, n))


def moe_forward_noalloc(desc, x, Wr, bias, W_gate_up, W_down, Wsh_gate_up, Wsh_down, y, topk_idx_out=None,
                        topk_w_out=None, stream=None):
    """moe_forward on the library's built-in 16 MiB scratch instead of a caller workspace."""
    _check("moe_forward_noalloc", lib().moe_forward_noalloc(
        ctypes.byref(desc), _p(x), _p(Wr), _p(bias), _p(W_gate_up), _p(W_down), _p(Wsh_gate_up), _p(Wsh_down),
        _p(y), _p(topk_idx_out), _p(topk_w_out), _stream(stream)))


def moe_forward_with_ids(desc, x, topk_idx, topk_w, W_gate_up, W_down, Wsh_gate_up, Wsh_down, y, ws, stream=None):
    """The layer with caller-supplied routing (routing replay / static benchmark routing)."""
    _check("moe_forward_with_ids", lib().moe_forward_with_ids(
        ctypes.byref(desc), _p(x), _p(topk_idx), _p(topk_w), _p(W_gate_up), _p(W_down), _p(Wsh_gate_up),
        _p(Wsh_down), _p(y), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_ep_pack(desc, x, topk_w, slot_of, x_send, w_send, stream=None):
    _check("moe_ep_pack", lib().moe_ep_pack(ctypes.byref(desc), _p(x), _p(topk_w), _p(slot_of), _p(x_send),
                                            _p(w_send), _stream(stream)))


def moe_ep_experts(desc, ep_ranks, recv_counts, x_recv, w_recv, W_gate_up, W_down, out, ws, stream=None):
    _check("moe_ep_experts", lib().moe_ep_experts(
        ctypes.byref(desc), int(ep_ranks), _p(recv_counts), _p(x_recv), _p(w_recv), _p(W_gate_up), _p(W_down),
        _p(out), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def moe_shared_expert(desc, x, Wsh_gate_up, Wsh_down, out, ws, stream=None):
    _check("moe_shared_expert", lib().moe_shared_expert(
        ctypes.byref(desc), _p(x), _p(Wsh_gate_up), _p(Wsh_down), _p(out), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))


def moe_host_workspace_size(desc: LayerDesc) -> int:
    out = ctypes.c_size_t(0)
    _check("moe_host_workspace_size", lib().moe_host_workspace_size(ctypes.byref(desc), ctypes.byref(out)))
    return out.value


def moe_forward_host(desc, n_batches, x_host, Wr, bias, W_gate_up, W_down, Wsh_gate_up, Wsh_down, y_host, ws,
                     stream=None, W_gate_up_scale=None, W_down_scale=None):
    _check("moe_forward_host", lib().moe_forward_host(
        ctypes.byref(desc), int(n_batches), _p(x_host), _p(Wr), _p(bias), _p(W_gate_up), _p(W_gate_up_scale),
        _p(W_down), _p(W_down_scale), _p(Wsh_gate_up), _p(Wsh_down), _p(y_host), _p(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)))
