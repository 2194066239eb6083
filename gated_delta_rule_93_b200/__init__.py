"""Gated delta-rule sequence mixer for NVIDIA B200 (sm_100a).

The computation lives in ``libgdr.so`` (CUDA kernels behind the C ABI in
``include/gdr.h``); ``binding`` is a ctypes front-end with the same names.
Importing this package does not load the library; the first call does.
"""
from .binding import (  # noqa: F401
    GdrError,
    chunk_bwd,
    chunk_bwd_workspace_bytes,
    chunk_fwd,
    chunk_fwd_gla,
    chunk_fwd_prologue,
    chunk_fwd_kernel_launches,
    chunk_fwd_segmented,
    chunk_fwd_varlen,
    chunk_fwd_workspace_bytes,
    dplr_fwd,
    device_status,
    lib,
    status_string,
    step,
)

__all__ = ["chunk_bwd", "chunk_bwd_workspace_bytes", "chunk_fwd", "chunk_fwd_gla", "chunk_fwd_prologue", "chunk_fwd_kernel_launches", "chunk_fwd_segmented", "chunk_fwd_varlen",
           "chunk_fwd_workspace_bytes", "dplr_fwd", "step", "device_status", "lib", "status_string",
           "GdrError"]
