"""Host-only checks of the C ABI: the library loads without a GPU, exports every
entry point that include/*.h declares, and rejects bad arguments before touching
the device (no kernel is launched by any call here)."""
import ctypes
import glob
import os
import re

import pytest

import sparse_moe_layer_biased_b200 as moe
from sparse_moe_layer_biased_b200 import _abi
from sparse_moe_layer_biased_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src))
    return names


def test_header_declares_the_binding_exports():
    assert declared_symbols() == set(_abi.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_status_strings():
    assert moe.moe_status_string(0) == "ok"
    assert moe.moe_status_string(3) == "workspace too small"
    assert moe.moe_status_string(99) == "unknown status"


def _desc(**kw):
    d = _abi.desc_of(WORKLOADS["tiny"])
    for k, v in kw.items():
        setattr(d, k, v)
    return d


FAKE = 1 << 20  # non-null, 16-byte aligned; never dereferenced because validation fails first


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), 1), (dict(k=17), 1), (dict(k=33, E=64), 1), (dict(T=-1), 1), (dict(H=0), 1),
    (dict(scale=float("nan")), 1), (dict(limit_routed=-1.0), 1), (dict(norm_expert_weight=2), 1),
    (dict(H=192), 2), (dict(I=96), 2), (dict(Is=32), 2), (dict(E=513, k=8), 2),
])
def test_bad_descriptors_rejected(kw, status):
    L = moe.lib()
    d = _desc(**kw)
    out = ctypes.c_size_t(0)
    assert L.moe_workspace_size(ctypes.byref(d), ctypes.byref(out)) == status
    assert L.moe_router(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == status
    assert L.moe_forward(ctypes.byref(d), *([FAKE] * 8), None, None, FAKE, 1 << 40, None) == status


def test_null_and_misaligned_pointers():
    L = moe.lib()
    d = _desc()
    assert L.moe_router(None, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert L.moe_router(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert L.moe_router(ctypes.byref(d), FAKE + 8, FAKE, FAKE, FAKE, FAKE, None, None) == 2
    assert L.moe_permute(ctypes.byref(d), FAKE, None, FAKE, FAKE, FAKE, None) == 1
    assert L.moe_combine(ctypes.byref(d), FAKE, FAKE, FAKE + 4, None) == 2
    args = [FAKE] * 8
    args[4] = None
    assert L.moe_forward(ctypes.byref(d), *args, None, None, FAKE, 1 << 40, None) == 1


def test_workspace_too_small_rejected():
    L = moe.lib()
    d = _desc()
    need = moe.moe_workspace_size(d)
    assert need > 0
    assert L.moe_forward(ctypes.byref(d), *([FAKE] * 8), None, None, FAKE, need - 1, None) == 3
    assert L.moe_expert_ffn(ctypes.byref(d), *([FAKE] * 10), FAKE, need - 1, None) == 3


def test_zero_tokens_is_a_no_op():
    L = moe.lib()
    d = _desc(T=0)
    need = moe.moe_workspace_size(d)
    assert L.moe_forward(ctypes.byref(d), *([FAKE] * 8), None, None, FAKE, need, None) == 0
    assert L.moe_router(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 0


def test_workspace_grows_with_tokens_and_determinism():
    s = WORKLOADS["step35_prefill"]
    a = moe.moe_workspace_size(_abi.desc_of(s))
    b = moe.moe_workspace_size(_abi.desc_of(s, T=2 * s.T))
    c = moe.moe_workspace_size(_abi.desc_of(s, deterministic=True))
    assert b > a and c - a >= (s.T * s.k + s.T) * s.H * 4


def test_wait_limit_roundtrip():
    old = moe.moe_set_wait_limit_ns(5_000_000)
    assert moe.moe_set_wait_limit_ns(old) == 5_000_000
    assert moe.moe_set_wait_limit_ns(old) == old


def test_stage_events_validation():
    L = moe.lib()
    arr = (ctypes.c_void_p * 2)(FAKE, None)
    assert L.moe_set_stage_events(arr, 2) == 1
    assert L.moe_set_stage_events(None, 1) == 1
    assert L.moe_set_stage_events(arr, 8) == 1
    assert L.moe_set_stage_events(None, 0) == 0


def test_with_ids_validation():
    L = moe.lib()
    d = _desc()
    need = moe.moe_workspace_size(d)
    args = [FAKE] * 8
    assert L.moe_forward_with_ids(ctypes.byref(d), *args, FAKE, need - 1, None) == 3
    args[1] = None
    assert L.moe_forward_with_ids(ctypes.byref(d), *args, FAKE, need, None) == 1
    args = [FAKE] * 8
    args[0] = FAKE + 2
    assert L.moe_forward_with_ids(ctypes.byref(d), *args, FAKE, need, None) == 2
    assert L.moe_forward_with_ids(ctypes.byref(_desc(T=0)), *([None] * 9), 0, None) == 0


def test_fp8_validation():
    L = moe.lib()
    d = _desc()
    assert d.I % 128 == 0
    need = moe.moe_workspace_size(d)
    args = [FAKE] * 10  # x, Wr, bias, codes / scales (gate_up, down), shared gate_up, shared down, y
    tail = [None, None, FAKE]
    assert L.moe_forward_fp8(ctypes.byref(d), *args, *tail, need - 1, None) == 3
    a = list(args)
    a[4] = None  # gate_up scales
    assert L.moe_forward_fp8(ctypes.byref(d), *a, *tail, need, None) == 1
    a = list(args)
    a[5] = FAKE + 8  # down codes not 16-byte aligned
    assert L.moe_forward_fp8(ctypes.byref(d), *a, *tail, need, None) == 2
    a = list(args)
    a[6] = FAKE + 2  # down scales not 4-byte aligned
    assert L.moe_forward_fp8(ctypes.byref(d), *a, *tail, need, None) == 2
    # I must be a multiple of 128 (gate and up rows start scale blocks), even with T = 0
    assert L.moe_forward_fp8(ctypes.byref(_desc(I=192)), *args, *tail, need, None) == 2
    assert L.moe_forward_fp8(ctypes.byref(_desc(T=0)), *([None] * 13), 0, None) == 0


def test_backward_validation():
    L = moe.lib()
    d = _desc()
    assert d.I % 128 == 0 and d.Is % 128 == 0
    need = moe.moe_backward_workspace_size(d)
    assert need > 0
    args = [FAKE] * 15  # x .. dWsh_down
    assert L.moe_backward(ctypes.byref(d), *args, FAKE, need - 1, None) == 3
    a = list(args)
    a[8] = None  # dy
    assert L.moe_backward(ctypes.byref(d), *a, FAKE, need, None) == 1
    a = list(args)
    a[9] = FAKE + 4  # dx misaligned
    assert L.moe_backward(ctypes.byref(d), *a, FAKE, need, None) == 2
    assert L.moe_backward(ctypes.byref(_desc(I=192)), *args, FAKE, need, None) == 2
    assert L.moe_backward(ctypes.byref(_desc(T=0)), *([None] * 16), 0, None) == 0


def test_ep_validation():
    L = moe.lib()
    d = _desc()
    # pack: null and misaligned pointers, empty call
    assert L.moe_ep_pack(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, None) == 1
    assert L.moe_ep_pack(ctypes.byref(d), FAKE + 2, FAKE, FAKE, FAKE, FAKE, None) == 2
    assert L.moe_ep_pack(ctypes.byref(_desc(T=0)), *([None] * 6)) == 0
    # owner side: k must be 1, ranks in 1..64, count table at most 8192 entries
    dl = _desc(k=1)
    need = moe.moe_workspace_size(dl)
    args = [FAKE] * 7
    assert L.moe_ep_experts(ctypes.byref(_desc(k=2)), 2, *args, need, None) == 1
    assert L.moe_ep_experts(ctypes.byref(dl), 0, *args, need, None) == 1
    assert L.moe_ep_experts(ctypes.byref(dl), 65, *args, need, None) == 1
    assert L.moe_ep_experts(ctypes.byref(_desc(k=1, E=512)), 64, *args, need, None) == 2
    assert L.moe_ep_experts(ctypes.byref(dl), 2, *args, need - 1, None) == 3
    a = list(args)
    a[0] = None  # recv_counts
    assert L.moe_ep_experts(ctypes.byref(dl), 2, *a, need, None) == 1
    a = list(args)
    a[1] = FAKE + 4  # x_recv not 16-byte aligned
    assert L.moe_ep_experts(ctypes.byref(dl), 2, *a, need, None) == 2
    assert L.moe_ep_experts(ctypes.byref(_desc(T=0, k=1)), 2, *([None] * 7), 0, None) == 0
    # shared expert alone
    need = moe.moe_workspace_size(d)
    assert L.moe_shared_expert(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, None) == 3
    assert L.moe_shared_expert(ctypes.byref(d), FAKE, None, FAKE, FAKE, FAKE, need, None) == 1
    assert L.moe_shared_expert(ctypes.byref(d), FAKE, FAKE, FAKE + 8, FAKE, FAKE, need, None) == 2
    assert L.moe_shared_expert(ctypes.byref(_desc(T=0)), *([None] * 5), 0, None) == 0


def test_forward_host_validation():
    L = moe.lib()
    d = _desc()
    need = moe.moe_host_workspace_size(d)
    assert need > moe.moe_workspace_size(d)
    # x_host, Wr, bias, W_gate_up, W_gate_up_scale, W_down, W_down_scale, Wsh_gate_up, Wsh_down, y_host, ws
    args = [FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE, FAKE, FAKE]
    assert L.moe_forward_host(ctypes.byref(d), -1, *args, need, None) == 1
    assert L.moe_forward_host(ctypes.byref(d), 2, *args, need - 1, None) == 3
    a = list(args)
    a[9] = None  # y_host
    assert L.moe_forward_host(ctypes.byref(d), 2, *a, need, None) == 1
    a = list(args)
    a[10] = FAKE + 8  # workspace not 16-byte aligned
    assert L.moe_forward_host(ctypes.byref(d), 2, *a, need, None) == 2
    a = list(args)
    a[4] = FAKE  # one FP8 scale array without the other
    assert L.moe_forward_host(ctypes.byref(d), 2, *a, need, None) == 1
    assert L.moe_forward_host(ctypes.byref(d), 0, *([None] * 11), 0, None) == 0
    assert L.moe_forward_host(ctypes.byref(_desc(T=0)), 3, *([None] * 11), 0, None) == 0
