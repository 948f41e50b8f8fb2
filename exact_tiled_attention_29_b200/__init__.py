"""Exact attention forward pass (FlashAttention-2 style) for NVIDIA B200, sm_100a.

The compute path is the C-ABI library ``libfa2.so`` (``include/fa2.h``); the
binding in ``_binding`` is loaded on first use of any of its names and raises
if the library has not been built.  ``inputs`` (seeded synthetic workloads)
does not load the library.
"""

_BINDING_NAMES = {
    "fa2_forward", "fa2_forward_local", "fa2_forward_ws", "fa2_backward", "fa2_backward_local",
    "fa2_backward_workspace_size", "attention_backward", "fa2_forward_static_ws", "fa2_workspace_size",
    "fa2_streamk_plan", "fa2_persistent_plan", "FA2_STATIC_WS_BYTES", "fa2_forward_auto",
    "fa2_schedule_choice",
    "alloc_workspace", "fa2_status_string", "fa2_debug_status", "fa2_selftest_timeout",
    "fa2_num_blocks", "fa2_launch_plan", "attention", "FA2Error", "LIB_PATH", "FA2_OK",
    "STATUS_NAMES", "SITE_NAMES", "FA2_SITE_SELFTEST",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
