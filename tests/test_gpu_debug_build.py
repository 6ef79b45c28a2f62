"""The debug build (libmoe_b200_debug.so, MOE_DEBUG): device-side range checks of every
index the kernels read from device data, reported by moe_check_device() as
MOE_ERR_DEVICE_BOUNDS instead of a fault.

1. The small parity shapes (router, permutation, forward in both modes, ties, hot and
   empty experts, replayed routing) run through the debug library in a child process
   (MOE_B200_DEBUG=1) against the CPU oracle; the parity module checks the device error
   word after its tests, so any failed range check fails the run.
2. A check does fire: moe_combine given one slot index past the routed slots (T*k + 1, a
   row that still lies inside the o_perm allocation, so even a build without checks would
   read valid memory) reports MOE_ERR_DEVICE_BOUNDS through the debug library.
"""
import os
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "sparse_moe_layer_biased_b200", "libmoe_b200_debug.so")

pytestmark = pytest.mark.gpu


def _child(args, timeout=1200):
    env = dict(os.environ, MOE_B200_DEBUG="1")
    return subprocess.run([sys.executable, *args], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not os.path.exists(DEBUG_LIB):
        pytest.fail(f"{DEBUG_LIB} is not built; run __graft_entry__.build()")


def test_small_parity_shapes_pass_the_range_checks():
    r = _child(["-m", "pytest", "tests/test_gpu_parity.py", "tests/test_gpu_fp8.py", "-m", "gpu and not slow",
                "-q", "-x", "-p", "no:cacheprovider"])
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout


def test_a_slot_past_the_routed_rows_is_reported():
    code = textwrap.dedent("""
        import torch
        from sparse_moe_layer_biased_b200 import _abi
        from sparse_moe_layer_biased_b200.inputs import LayerShape
        assert _abi.DEBUG and _abi.LIB_PATH.endswith("libmoe_b200_debug.so")
        sh = LayerShape("c", T=8, H=128, E=4, k=2, I=64, Is=64)
        d = _abi.desc_of(sh, deterministic=True)
        o_perm = torch.zeros((sh.T * sh.k + sh.T, sh.H), device="cuda")
        slot = torch.arange(sh.T * sh.k, dtype=torch.int32, device="cuda").view(sh.T, sh.k).contiguous()
        y = torch.empty((sh.T, sh.H), device="cuda")
        _abi.moe_combine(d, o_perm, slot, y)
        assert _abi.lib().moe_check_device() == 0
        slot[3, 1] = sh.T * sh.k + 1   # past the routed slots, inside the allocation
        _abi.moe_combine(d, o_perm, slot, y)
        assert _abi.lib().moe_check_device() == 6   # MOE_ERR_DEVICE_BOUNDS
        assert _abi.lib().moe_check_device() == 0   # reported once, then cleared
        print("range check reported")
        """)
    r = _child(["-c", code], timeout=300)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "range check reported" in r.stdout
