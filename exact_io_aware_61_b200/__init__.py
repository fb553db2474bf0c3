"""Exact IO-aware tiled attention for NVIDIA B200 (sm_100a).

``forward`` / ``backward`` run the hand-written CUDA kernels of
``libfa_b200.so`` through its C ABI (``include/fa.h``); the library is loaded
on first use and its absence is an error, never a fallback.
"""

from ._lib import (  # noqa: F401
    EXPORTED,
    FA_BF16,
    FA_ERR_CUDA,
    FA_ERR_INVALID,
    FA_ERR_TIMEOUT,
    FA_ERR_UNSUPPORTED,
    FA_ERR_WORKSPACE,
    FA_F32,
    FA_OK,
    LIB_PATH,
    FAError,
    backward,
    backward_bnhd,
    backward_varlen,
    fa_bwd,
    fa_bwd_main,
    fa_bwd_dq,
    fa_bwd_noalloc,
    fa_bwd_partial,
    fa_bwd_prep,
    fa_bwd_varlen,
    fa_bwd_varlen_workspace_size,
    fa_bwd_workspace_size,
    fa_fwd,
    fa_f32_to_bf16,
    fa_fwd_kvcache,
    fa_fwd_partial,
    fa_fwd_varlen,
    fa_fwd_kvcache_workspace_size,
    fa_last_device_status,
    fa_merge_partials,
    fa_selftest_wait_timeout,
    fa_set_wait_timeout_ns,
    forward,
    forward_bnhd,
    forward_kvcache,
    forward_varlen,
    load,
    status_string,
)
