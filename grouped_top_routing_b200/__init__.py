"""B200-native (sm_100a) grouped top-k MoE feed-forward block.

The compute lives in ``libmoe.so`` (hand-written CUDA behind a C ABI, declared
in ``include/moe.h``); ``grouped_top_routing_b200.moe`` is a thin ctypes
binding with the same entry-point names. Importing the binding raises if the
library has not been built: there is no fallback.
"""

_BINDING_NAMES = (
    "MoeConfig", "MoeError", "Workspace", "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine",
    "moe_forward", "moe_workspace_size", "moe_router_logits", "lib", "library_path", "config_from_workload",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import moe
        return getattr(moe, name)
    raise AttributeError(name)
