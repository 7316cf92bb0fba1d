"""Selective-SSM scan and single-token state update for NVIDIA B200 (sm_100a).

The computation lives in ``libmamba_ssm.so`` (hand-written CUDA behind the C
ABI of ``include/mamba_ssm.h``); ``ops`` is its ctypes binding and ``inputs``
the seeded synthetic workloads.  Besides the scan and the update, the library
holds the scan over host buffers, the block's short causal convolution, the
scan's backward pass and the Mamba-2 layer (scalar A per head) on the tensor
cores.
"""
from . import inputs  # noqa: F401
from .ops import (  # noqa: F401
    MambaError, causal_conv1d_fwd, causal_conv1d_update, device_status, scan_host_workspace_bytes,
    scan_plan, scan_workspace_bytes, selective_scan_fwd, selective_scan_fwd_host,
    selective_state_update, ssd_chunk_scan_fwd, status_string, version,
)

__all__ = [
    "inputs", "MambaError", "causal_conv1d_fwd", "causal_conv1d_update", "device_status",
    "scan_host_workspace_bytes", "scan_plan", "scan_workspace_bytes", "selective_scan_fwd",
    "selective_scan_fwd_host", "selective_state_update", "ssd_chunk_scan_fwd", "status_string",
    "version",
]
