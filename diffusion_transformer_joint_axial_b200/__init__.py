"""Qwen-Image-2.1 joint-attention hot path for B200 (sm_100a).

3D axial RoPE (bands 16/56/56, centred image grids), the Block-Causal mask
and the Prefix KV Cache, computed by the CUDA kernels of ``libqi21.so``
behind a C ABI (``include/qi21.h``).  This package is the thin Python
binding: it marshals torch tensors into that ABI and nothing else.
"""

from ._binding import (HEAD_DIM, LIB_PATH, QI21Error, Segment, alloc_cache, attn_cached, attn_full,
                       cached_workspace_size, full_workspace_size, interleave_gate_up, launch_count, linear,
                       linear_residual, linear_swiglu,
                       load_library, new_workspace, rmsnorm, rope_positions, rope_table, rope_table_size,
                       selftest_wait_timeout, swiglu, workspace_status)
from . import denoise
from .steploop import DenoiseLoop

__all__ = ["DenoiseLoop", "HEAD_DIM", "LIB_PATH", "QI21Error", "Segment", "alloc_cache", "attn_cached",
           "attn_full", "cached_workspace_size", "full_workspace_size", "interleave_gate_up", "launch_count",
           "linear", "linear_residual", "linear_swiglu", "load_library", "new_workspace", "rmsnorm", "rope_positions", "rope_table", "rope_table_size",
           "selftest_wait_timeout", "swiglu", "workspace_status"]
