"""libssd: the scalar-decay selective state-space layer (Mamba-2 SSD) on B200.

The compute lives in libssd.so (hand-written sm_100a CUDA behind a C ABI,
include/ssd.h); this package is its Python binding. Importing the package does
not load the library; the first call does, and fails loudly if it is missing.
"""
from .sp import sp_forward
from .ssd import (CHUNKS, HostForward, PreparedCall, SSDError, launch_count, make_dims, make_options,
                  prepare_forward, prepare_step, profile_begin, profile_end, ssd_abi_version,
                  ssd_backward, ssd_device_status, ssd_forward, ssd_forward_ex, ssd_forward_state,
                  ssd_forward_workspace_size, ssd_last_error, ssd_selective_scan,
                  ssd_set_wait_limit, ssd_state_chain, ssd_step,
                  ssd_step_ex)

__all__ = ["CHUNKS", "HostForward", "PreparedCall", "SSDError", "launch_count", "make_dims", "make_options",
           "prepare_forward", "prepare_step", "profile_begin", "profile_end", "ssd_abi_version", "ssd_backward",
           "ssd_device_status", "ssd_forward", "ssd_forward_ex", "ssd_forward_state",
           "ssd_forward_workspace_size", "ssd_last_error", "ssd_selective_scan",
           "ssd_set_wait_limit", "ssd_state_chain", "sp_forward",
           "ssd_step", "ssd_step_ex"]
