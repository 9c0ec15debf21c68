"""Exact scaled-dot-product attention for B200 (sm_100a).

The compute lives in ``libfa.so`` (hand-written CUDA, C ABI in include/fa.h);
``binding`` marshals arguments to it.  Importing the package does not load
the library; the first call does, and fails loudly when it is missing.
"""
from .binding import (  # noqa: F401
    FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_ARCH, FA_ERR_CUDA,
    FA_ERR_TIMEOUT, FaError, lib, lib_path, fa_fwd, fa_fwd_pair, fa_bwd, fa_fwd_f32, fa_bwd_f32,
    fa_fwd_splitkv, fa_fwd_splitkv_num_splits, fa_fwd_splitkv_workspace_size,
    fa_fwd_fp8, forward_fp8,
    fa_fwd_dropout, fa_bwd_dropout, forward_dropout, backward_dropout,
    fa_bwd_workspace_size, fa_bwd_prep, fa_bwd_dkdv, fa_bwd_dq, fa_device_status,
    fa_wait_selftest, fa_strerror, forward, forward_splitkv, backward,
)
