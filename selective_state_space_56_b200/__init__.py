"""B200-native selective scan (S6): fused forward scan, its backward, the
single-token state update, and the causal conv1d + SiLU producing the scan's input
(forward, decode step and backward).

The compute lives in hand-written sm_100a CUDA kernels behind a C ABI
(``include/mamba_s6.h``, built into ``libmamba_s6.so`` in this package by
``python -m selective_state_space_56_b200.build``).  The Python functions here
only marshal torch tensors into that ABI.
"""
from .ops import (  # noqa: F401
    MambaError,
    causal_conv1d_bwd,
    causal_conv1d_fwd,
    causal_conv1d_update,
    check_device_error,
    load_library,
    selective_scan_bwd,
    selective_scan_bwd_workspace_size,
    selective_scan_fwd,
    selective_scan_workspace_size,
    selective_state_update,
    status_string,
)
