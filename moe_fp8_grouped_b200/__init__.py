"""FP8 grouped matmul (gmm forward, gmm dlhs, tgmm drhs) for MoE expert MLPs
on B200 (sm_100a).

The compute runs in the CUDA library ``libgmm_fp8.so`` (C-ABI declared in
``include/gmm_fp8.h``); ``ops`` is a thin ctypes binding with the same names.
The library is loaded on first use and a missing library raises an error:
there is no CPU fallback.
"""
# populated once ops.py exists
# from .ops import (  # noqa: F401
#     GmmError, gmm_fwd, gmm_dlhs, tgmm_drhs, gmm_quantize, gmm_quantize_rhs, gmm_plan, gmm_workspace_bytes,
#     gmm_read_device_status, gmm_status_string, QRule, DType,
# )
