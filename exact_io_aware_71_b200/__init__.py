"""Exact IO-aware tiled attention for NVIDIA B200 (sm_100a).

The compute lives in ``libfa.so`` (hand-written CUDA, C ABI in
``include/fa.h``); this package is its ctypes binding plus the seeded input
generators used by the tests and the benchmark.
"""
from .binding import (  # noqa: F401
    FA_OK,
    FaError,
    backward,
    fa_bwd,
    fa_bwd_stage,
    fa_bwd_strided,
    fa_fwd_strided,
    fa_fwd_block_sparse,
    fa_bwd_block_sparse,
    fa_fwd_residual,
    fa_bwd_residual,
    MASK_BLOCK,
    fa_fwd_varlen,
    fa_bwd_varlen,
    fa_bwd_varlen_workspace_size,
    forward_varlen,
    backward_varlen,
    FaStrides,
    strides_of,
    fa_bwd_workspace_size,
    fa_device_status,
    fa_fwd,
    fa_status_string,
    forward,
    load,
)
