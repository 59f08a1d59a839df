"""HiLS (Hierarchical Landmark Sparse) attention forward pass for B200 (sm_100a).

The computation runs in the CUDA kernels of libhils.so behind the C ABI in include/hils.h;
`binding` marshals torch tensors into that ABI and `workloads` draws seeded synthetic inputs.
"""
from .binding import (HilsError, Params, chunk_attn, device_status, forward, fuse, lib,
                      make_params, select, version, workspace, workspace_size)

__all__ = ["HilsError", "Params", "chunk_attn", "device_status", "forward", "fuse", "lib",
           "make_params", "select", "version", "workspace", "workspace_size"]
