"""B200-native exact attention forward (FlashAttention-style), C-ABI library + thin binding.

The compute path is the shared library ``libfa_b200.so`` built from ``csrc/``
(hand-written sm_100a CUDA: TMA, mbarrier pipelines, tcgen05 MMAs into TMEM).
This package only marshals arguments into it.  Importing the package does not
load the library; the first call does, and raises if it is missing -- there is
no fallback of any kind.
"""
from .binding import (  # noqa: F401
    FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED, FA_ERR_CUDA,
    FA_ERR_NO_DEVICE, FA_ERR_DEVICE_TIMEOUT, FaError, attention, fa_fwd,
    fa_fwd_host, fa_fwd_host_workspace_size, fa_bwd, fa_bwd_workspace_size, fa_fwd_splitkv, fa_fwd_splitkv_noalloc,
    fa_fwd_splitkv_workspace_size, fa_fwd_window, fa_fwd_bias, fa_fwd_bias_table, fa_fwd_fp8, fa_fwd_varlen,
    fa_splitkv_num_splits, fa_get_device_status, fa_selftest_wait_timeout,
    fa_selftest_fwd_timeout, fa_selftest_bwd_timeout,
    fa_status_string, fa_last_error,
    fa_version, library_path, load_library,
)
