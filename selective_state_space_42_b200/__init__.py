"""libselscan: the Mamba-1 selective scan, its gradient, its single-token
state update and the scalar-A-per-head (Mamba-2) scan in chunked form, as
hand-written CUDA for B200 (sm_100a) behind a C ABI (include/selscan.h).

The Python functions below are a thin ctypes binding with the same names as
the C entry points; see ``selscan.py``.
"""
from .selscan import (LIB_PATH, SELSCAN_BF16, SELSCAN_F32, SELSCAN_MAX_DSTATE,
                      SELSCAN_MAX_DSTATE_BWD,
                      SELSCAN_NOALLOC_WORKSPACE_BYTES,
                      SelscanError, SelscanUnavailable, load_library,
                      selscan_bwd, selscan_bwd_workspace_bytes,
                      selscan_device_status, selscan_fwd, selscan_fwd_noalloc,
                      selscan_fwd_plan,
                      selscan_last_cuda_error,
                      selscan_ssd_fwd, selscan_state_update, selscan_status_string)

__all__ = ["selscan_bwd", "selscan_bwd_workspace_bytes", "selscan_device_status", "selscan_fwd", "selscan_fwd_noalloc", "selscan_fwd_plan", "selscan_state_update", "selscan_ssd_fwd", "selscan_status_string",
           "selscan_last_cuda_error", "load_library", "SelscanError",
           "SelscanUnavailable", "LIB_PATH", "SELSCAN_F32", "SELSCAN_BF16",
           "SELSCAN_MAX_DSTATE", "SELSCAN_MAX_DSTATE_BWD", "SELSCAN_NOALLOC_WORKSPACE_BYTES"]
