"""ctypes wrapper of the CPU oracle (oracle/moe_oracle.c).

TEST INFRASTRUCTURE ONLY: tests, the package smoke check and the benchmark's CPU
baseline leg use it; the product path never imports it. Inputs are numpy arrays;
bf16 tensors are passed as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None

_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_router_logits.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _u16p, _u16p, _f32p]
        L.oracle_router_select.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _f32p, _f32p,
                                           ctypes.c_float, ctypes.c_int, _i32p, _vp, _vp, _vp, _vp]
        L.oracle_permute.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, _i32p, _i32p, _i32p,
                                     _i32p, _i32p]
        L.oracle_permute.restype = ctypes.c_int
        L.oracle_swiglu_hidden.argtypes = [ctypes.c_int, ctypes.c_int, _u16p, _u16p, ctypes.c_double, _f64p]
        L.oracle_swiglu_mlp.argtypes = [ctypes.c_int, ctypes.c_int, _u16p, _u16p, _u16p, ctypes.c_double,
                                        _f64p, _f64p]
        L.oracle_forward_tokens.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                            ctypes.c_float, ctypes.c_float, _u16p, _u16p, _f32p,
                                            ctypes.POINTER(_vp), ctypes.POINTER(_vp), _u16p, _u16p, _f64p,
                                            _i32p, _f64p, _f32p]
        L.oracle_forward_tokens.restype = ctypes.c_int
        L.oracle_forward_given_routing.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                                   _u16p, _i32p, _f32p, ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                                   _u16p, _u16p, _f64p]
        L.oracle_forward_given_routing.restype = ctypes.c_int
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_dequant_block128.argtypes = [ctypes.c_int64, ctypes.c_int64, _u8p, _f32p, _f32p]
        L.oracle_experts_f32w.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_float, ctypes.c_float, _u16p, _i32p, _f64p,
                                          ctypes.POINTER(_vp), ctypes.POINTER(_vp), _u16p, _u16p, _f64p]
        L.oracle_experts_f32w.restype = ctypes.c_int
        L.oracle_backward.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                      _u16p, _u16p, _f32p, _u16p, _u16p, _u16p, _u16p, _f32p, _f64p, _f64p, _f64p,
                                      _f64p, _f64p, _f64p, _i32p, _f64p, _f64p]
        L.oracle_backward.restype = ctypes.c_int
        L.oracle_forward_dense.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                           ctypes.c_float, ctypes.c_float, _u16p, _u16p, _f32p, _u16p,
                                           _u16p, _u16p, _u16p, _f64p]
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def _ptr(a):
    return a.ctypes.data_as(_vp) if a is not None else None


def router_logits(x, Wr):
    x, Wr = _u16(x), _u16(Wr)
    T, H = x.shape
    E = Wr.shape[0]
    out = np.empty((T, E), np.float32)
    lib().oracle_router_logits(T, H, E, x, Wr, out)
    return out


def router_select(logits, bias, k, scale=3.0, norm=True):
    logits = np.ascontiguousarray(logits, np.float32)
    bias = np.ascontiguousarray(bias, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w32 = np.empty((T, k), np.float32)
    w64 = np.empty((T, k), np.float64)
    margin = np.empty((T,), np.float32)
    scores = np.empty((T, E), np.float32)
    lib().oracle_router_select(T, E, k, logits, bias, scale, int(bool(norm)), idx, _ptr(w32), _ptr(w64),
                               _ptr(margin), _ptr(scores))
    return {"idx": idx, "w": w64, "w32": w32, "margin": margin, "scores": scores}


def router(x, Wr, bias, k, scale=3.0, norm=True):
    """Full routing step: fp32 logits, sigmoid, biased top-k, weights, margin."""
    logits = router_logits(x, Wr)
    out = router_select(logits, bias, k, scale, norm)
    out["logits"] = logits
    return out


def permute(idx, E):
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E + 1, np.int32)
    offsets = np.empty(E + 2, np.int32)
    perm_token = np.empty(T * k + T, np.int32)
    slot_of = np.empty((T, k), np.int32)
    rc = lib().oracle_permute(T, k, E, idx, counts, offsets, perm_token, slot_of)
    if rc != 0:
        raise ValueError("expert id out of range")
    return {"counts": counts, "offsets": offsets, "perm_token": perm_token, "slot_of": slot_of}


def swiglu_hidden(x_row, Wgu, limit):
    x_row, Wgu = _u16(x_row), _u16(Wgu)
    H = x_row.shape[0]
    Iw = Wgu.shape[0] // 2
    out = np.empty(Iw, np.float64)
    lib().oracle_swiglu_hidden(H, Iw, x_row, Wgu, float(limit), out)
    return out


def swiglu_mlp(x_row, Wgu, Wd, limit):
    x_row, Wgu, Wd = _u16(x_row), _u16(Wgu), _u16(Wd)
    H = x_row.shape[0]
    Iw = Wgu.shape[0] // 2
    out = np.empty(H, np.float64)
    hid = np.empty(Iw, np.float64)
    lib().oracle_swiglu_mlp(H, Iw, x_row, Wgu, Wd, float(limit), out, hid)
    return out


def forward_tokens(x_rows, Wr, bias, experts, Wsh_gu, Wsh_d, *, k, scale=3.0, norm=True,
                   limit_routed=0.0, limit_shared=0.0):
    """Layer output for the given token rows.

    experts: mapping expert id -> (W_gate_up[e] [2I, H] uint16, W_down[e] [H, I] uint16);
    it must hold every expert the listed tokens select (others may be absent).
    Returns dict(y [n, H] float64, idx, w, margin).
    """
    x_rows, Wr = _u16(x_rows), _u16(Wr)
    bias = np.ascontiguousarray(bias, np.float32)
    n, H = x_rows.shape
    E = Wr.shape[0]
    keep = {}
    gu_ptrs = (_vp * E)()
    d_ptrs = (_vp * E)()
    I = None
    for e, (gu, d) in experts.items():
        gu, d = _u16(gu), _u16(d)
        keep[e] = (gu, d)
        gu_ptrs[e] = gu.ctypes.data
        d_ptrs[e] = d.ctypes.data
        I = gu.shape[0] // 2
    Wsh_gu, Wsh_d = _u16(Wsh_gu), _u16(Wsh_d)
    Is = Wsh_gu.shape[0] // 2
    if I is None:
        I = Is
    y = np.empty((n, H), np.float64)
    idx = np.empty((n, k), np.int32)
    w = np.empty((n, k), np.float64)
    margin = np.empty((n,), np.float32)
    rc = lib().oracle_forward_tokens(n, H, E, k, I, Is, scale, int(bool(norm)), limit_routed, limit_shared,
                                     x_rows, Wr, bias, gu_ptrs, d_ptrs, Wsh_gu, Wsh_d, y, idx, w, margin)
    del keep
    if rc != 0:
        raise ValueError("a selected expert's weights were not supplied")
    return {"y": y, "idx": idx, "w": w, "margin": margin}


def forward_given_routing(x_rows, idx, w, experts, Wsh_gu, Wsh_d, *, E, limit_routed=0.0, limit_shared=0.0):
    """Layer output for caller-supplied routing (ids [n, k] int32, weights [n, k] fp32).

    experts: mapping expert id -> (W_gate_up[e], W_down[e]) holding every id used.
    """
    x_rows = _u16(x_rows)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    n, H = x_rows.shape
    k = idx.shape[1]
    keep = {}
    gu_ptrs = (_vp * E)()
    d_ptrs = (_vp * E)()
    I = None
    for e, (gu, d) in experts.items():
        gu, d = _u16(gu), _u16(d)
        keep[e] = (gu, d)
        gu_ptrs[e] = gu.ctypes.data
        d_ptrs[e] = d.ctypes.data
        I = gu.shape[0] // 2
    Wsh_gu, Wsh_d = _u16(Wsh_gu), _u16(Wsh_d)
    Is = Wsh_gu.shape[0] // 2
    if I is None:
        I = Is
    y = np.empty((n, H), np.float64)
    rc = lib().oracle_forward_given_routing(n, H, E, k, I, Is, limit_routed, limit_shared, x_rows, idx, w,
                                            gu_ptrs, d_ptrs, Wsh_gu, Wsh_d, y)
    del keep
    if rc != 0:
        raise ValueError("a used expert's weights were not supplied")
    return y


def forward_dense(x, Wr, bias, W_gate_up, W_down, Wsh_gu, Wsh_d, *, k, scale=3.0, norm=True,
                  limit_routed=0.0, limit_shared=0.0):
    """Brute force: all experts on all tokens, mixed by a mask-weight matrix."""
    x, Wr, W_gate_up, W_down = _u16(x), _u16(Wr), _u16(W_gate_up), _u16(W_down)
    Wsh_gu, Wsh_d = _u16(Wsh_gu), _u16(Wsh_d)
    bias = np.ascontiguousarray(bias, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    I = W_gate_up.shape[1] // 2
    Is = Wsh_gu.shape[0] // 2
    y = np.empty((T, H), np.float64)
    lib().oracle_forward_dense(T, H, E, k, I, Is, scale, int(bool(norm)), limit_routed, limit_shared,
                               x, Wr, bias, W_gate_up, W_down, Wsh_gu, Wsh_d, y)
    return y


def forward_full(inp: dict, shape, *, limit_routed=None, limit_shared=None, scale=None, norm=None):
    """forward_tokens over every token of a drawn workload (small shapes only)."""
    from sparse_moe_layer_biased_b200.inputs import bf16_bits  # the shared input module
    gu = bf16_bits(inp["W_gate_up"])
    d = bf16_bits(inp["W_down"])
    experts = {e: (gu[e], d[e]) for e in range(shape.E)}
    return forward_tokens(
        bf16_bits(inp["x"]), bf16_bits(inp["Wr"]), inp["bias"].cpu().numpy(), experts,
        bf16_bits(inp["Wsh_gate_up"]), bf16_bits(inp["Wsh_down"]), k=shape.k,
        scale=shape.scale if scale is None else scale,
        norm=shape.norm_expert_weight if norm is None else norm,
        limit_routed=shape.limit_routed if limit_routed is None else limit_routed,
        limit_shared=shape.limit_shared if limit_shared is None else limit_shared)


def e4m3_values():
    """Value of every E4M3 code 0..255 (float64; NaN for the two NaN codes)."""
    return np.array([lib().oracle_e4m3_value(c) for c in range(256)], np.float64)


def dequant_block128(q, scale):
    """FP8 E4M3 matrix q [rows, cols] (uint8 codes) with 128x128 block scales
    scale [ceil(rows/128), ceil(cols/128)] -> fp32 weights."""
    q = np.ascontiguousarray(q, np.uint8)
    scale = np.ascontiguousarray(scale, np.float32)
    rows, cols = q.shape
    assert scale.shape == ((rows + 127) // 128, (cols + 127) // 128)
    out = np.empty((rows, cols), np.float32)
    lib().oracle_dequant_block128(rows, cols, q, scale, out)
    return out


def experts_f32w(x_rows, idx, w, experts, Wsh_gu, Wsh_d, *, E, limit_routed=0.0, limit_shared=0.0):
    """Expert part of the layer for a given routing (ids [n, k], weights [n, k] float64)
    with fp32 routed-expert weights: experts maps id -> (W_gate_up [2I, H] f32,
    W_down [H, I] f32); the shared expert is BF16 (uint16 bits)."""
    x_rows = _u16(x_rows)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    n, H = x_rows.shape
    k = idx.shape[1]
    keep = {}
    gu_ptrs = (_vp * E)()
    d_ptrs = (_vp * E)()
    I = None
    for e, (gu, d) in experts.items():
        gu = np.ascontiguousarray(gu, np.float32)
        d = np.ascontiguousarray(d, np.float32)
        keep[e] = (gu, d)
        gu_ptrs[e] = gu.ctypes.data
        d_ptrs[e] = d.ctypes.data
        I = gu.shape[0] // 2
    Wsh_gu, Wsh_d = _u16(Wsh_gu), _u16(Wsh_d)
    Is = Wsh_gu.shape[0] // 2
    if I is None:
        I = Is
    y = np.empty((n, H), np.float64)
    rc = lib().oracle_experts_f32w(n, H, E, k, I, Is, limit_routed, limit_shared, x_rows, idx, w, gu_ptrs,
                                   d_ptrs, Wsh_gu, Wsh_d, y)
    del keep
    if rc != 0:
        raise ValueError("a used expert's weights were not supplied")
    return y


def forward_fp8_tokens(x_rows, Wr, bias, Wgu_q, Wgu_s, Wd_q, Wd_s, Wsh_gu, Wsh_d, *, k, scale=3.0, norm=True,
                       limit_routed=0.0, limit_shared=0.0):
    """Layer output for the given token rows with FP8 E4M3 routed experts: routing as in
    router(), then the selected experts dequantized (dequant_block128) and applied with
    the BF16 shared expert. Wgu_q [E, 2I, H] / Wd_q [E, H, I] uint8 codes with block
    scales Wgu_s [E, 2I/128, H/128] / Wd_s [E, H/128, I/128]. Returns dict(y, idx, w, margin)."""
    r = router(x_rows, Wr, bias, k, scale, norm)
    E = Wgu_q.shape[0]
    experts = {int(e): (dequant_block128(Wgu_q[e], Wgu_s[e]), dequant_block128(Wd_q[e], Wd_s[e]))
               for e in np.unique(r["idx"])}
    y = experts_f32w(x_rows, r["idx"], r["w"], experts, Wsh_gu, Wsh_d, E=E, limit_routed=limit_routed,
                     limit_shared=limit_shared)
    return {"y": y, "idx": r["idx"], "w": r["w"], "margin": r["margin"]}


def backward(x, Wr, bias, W_gate_up, W_down, Wsh_gu, Wsh_d, dy, *, k, scale=3.0, norm=True, limit_routed=0.0,
             limit_shared=0.0):
    """Gradients of the layer for upstream gradient dy [T, H] (fp32): dict(dx [T, H], dWr [E, H],
    dW_gate_up [E, 2I, H], dW_down [E, H, I], dWsh_gate_up [2Is, H], dWsh_down [H, Is]) in
    float64, plus the forward's idx, w and dw = dLoss/dw [T, k]. The router bias gets no
    gradient (selection only). Stacked weights; small shapes only (one pass over all tokens)."""
    x, Wr, W_gate_up, W_down = _u16(x), _u16(Wr), _u16(W_gate_up), _u16(W_down)
    Wsh_gu, Wsh_d = _u16(Wsh_gu), _u16(Wsh_d)
    bias = np.ascontiguousarray(bias, np.float32)
    dy = np.ascontiguousarray(dy, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    I = W_gate_up.shape[1] // 2
    Is = Wsh_gu.shape[0] // 2
    out = {"dx": np.empty((T, H)), "dWr": np.empty((E, H)), "dW_gate_up": np.empty((E, 2 * I, H)),
           "dW_down": np.empty((E, H, I)), "dWsh_gate_up": np.empty((2 * Is, H)), "dWsh_down": np.empty((H, Is)),
           "idx": np.empty((T, k), np.int32), "w": np.empty((T, k)), "dw": np.empty((T, k))}
    lib().oracle_backward(T, H, E, k, I, Is, scale, int(bool(norm)), limit_routed, limit_shared, x, Wr, bias,
                          W_gate_up, W_down, Wsh_gu, Wsh_d, dy, out["dx"], out["dWr"], out["dW_gate_up"],
                          out["dW_down"], out["dWsh_gate_up"], out["dWsh_down"], out["idx"], out["w"], out["dw"])
    return out


__all__ = ["lib", "num_threads", "router_logits", "router_select", "router", "permute", "swiglu_hidden",
           "swiglu_mlp", "forward_tokens", "forward_given_routing", "forward_dense", "forward_full", "e4m3_values",
           "dequant_block128", "experts_f32w", "forward_fp8_tokens", "backward"]
