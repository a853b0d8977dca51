"""B200-native decode attention for Flint (sm_100a CUDA behind a C ABI).

The compute path lives in ``csrc/`` and is exported by ``libflint.so``; the
Python names here are a thin ctypes binding over that C ABI.  ``inputs``
generates the seeded synthetic workloads.
"""
_BINDING_NAMES = (
    "FlintError", "load_library", "flint_status_string", "flint_last_error",
    "flint_kv_bytes", "flint_qk_norm_rope", "flint_kv_append",
    "flint_attn_workspace_bytes", "flint_attn_decode", "flint_attn_stack",
    "flint_attn_stack_noalloc", "flint_attn_layers_serial",
    "flint_plan_items", "flint_plan_split", "KVCache", "StackLayer",
)

__all__ = list(_BINDING_NAMES) + ["inputs"]


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import flint
        return getattr(flint, name)
    raise AttributeError(name)
