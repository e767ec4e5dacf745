"""FP8 grouped matmul (gmm forward, gmm dlhs, tgmm drhs) for MoE expert MLPs
on B200 (sm_100a).

The compute runs in the CUDA library ``libgmm_fp8.so`` (C-ABI declared in
``include/gmm_fp8.h``); ``ops`` is a thin ctypes binding with the same names.
The library is loaded on first use and a missing library raises an error:
there is no CPU fallback.
"""
from .ops import (  # noqa: F401
    DType, GmmError, QRule, gmm_backward, gmm_chunk_capacity, gmm_dlhs, gmm_fwd, gmm_fwd_keep_lhs, gmm_fwd_swiglu,
    gmm_plan, gmm_quantize, gmm_quantize_rhs, gmm_quantize_rhs_blocks, gmm_read_device_status, gmm_selftest_timeout,
    gmm_set_tiles, gmm_set_wait_limit_ns, gmm_status_string, gmm_workspace_bytes, last_launch_count, profile_collect,
    profile_enable, tgmm_drhs, workspace,
)
