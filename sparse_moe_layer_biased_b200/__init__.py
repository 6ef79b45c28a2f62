"""B200 (sm_100a) forward and backward passes of the biased-sigmoid-routed MoE FFN layer.

The kernels live in libmoe_b200.so behind the C ABI of include/moe_b200.h; the
entry points are re-exported here under the same names (see _abi.py). MoeLayer
(layer.py) holds device weights and a workspace and calls moe_forward (or
moe_forward_fp8 for FP8 routed experts). The seeded
synthetic input generator is in inputs.py. Importing the package does not load the
library; the first call does, and raises if it is not built.
"""
_ABI = {"moe_status_string", "moe_workspace_size", "moe_router", "moe_permute", "moe_expert_ffn", "moe_combine",
        "moe_forward", "moe_check_device", "moe_set_wait_limit_ns", "moe_set_stage_events", "moe_forward_noalloc",
        "moe_forward_with_ids", "moe_forward_fp8", "moe_backward", "moe_backward_workspace_size", "moe_ep_pack",
        "moe_ep_experts", "moe_shared_expert", "moe_host_workspace_size", "moe_forward_host", "MoeError",
        "LayerDesc", "desc_of", "lib", "EXPORTS", "LIB_PATH"}


def __getattr__(name):
    if name in _ABI:
        from . import _abi

        return getattr(_abi, name)
    if name == "MoeLayer":
        from .layer import MoeLayer

        return MoeLayer
    if name == "EPMoeLayer":
        from .ep import EPMoeLayer

        return EPMoeLayer
    raise AttributeError(name)
