"""B200-native (sm_100a) information-form Kalman filter scan of Kalman Linear
Attention (KLA).

The compute path is the C-ABI CUDA library ``libkla.so`` (declared in
``include/kla.h``); :mod:`.api` is its thin ctypes binding and is imported on
first use, so that importing :mod:`.workloads` (seeded inputs) needs neither
torch nor the built library.
"""
_API_NAMES = {
    "scan_forward", "scan_step", "workspace_size", "new_workspace", "get_error",
    "set_wait_limit_ns", "debug_unset_flag_wait", "debug_stall_chunk", "chunk_tokens",
    "debug_force_forward_kernel", "forward_plan", "host_workspace_size",
    "KlaError", "lib", "load_library", "scan_forward_static",
    "scan_backward", "backward_workspace_size", "backward_plan", "debug_force_backward_kernel",
    "KalmanFilterScan", "kalman_filter", "layer_forward", "layer_workspace_size", "layer_step",
    "attention_weights", "scan_forward_lti", "lti_workspace_size", "lti_plan",
}


def __getattr__(name):
    if name in _API_NAMES:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
