"""Exact scaled-dot-product attention for NVIDIA B200 (sm_100a).

``O = softmax(scale * Q K^T [+ causal mask]) V`` and its gradient, computed tile
by tile with an online softmax so the N x N score and probability matrices
never reach HBM (FlashAttention-2, "Faster Attention with Better Parallelism
and Work Partitioning", abstract; iplexlaw FlashAttention-2 blog, "Tiling
preserves the attention calculation").

The compute lives in ``libfa_sm100.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/fa.h``).  This package is a thin binding: it
marshals torch tensors into pointers and sizes and calls the C entry points of
the same names.  There is no CPU fallback; when the library is missing, every
call raises.
"""
from .api import (  # noqa: F401
    FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED,
    FA_ERR_CUDA, FA_ERR_TIMEOUT, FaError, library, library_path,
    fa_fwd, fa_bwd, fa_bwd_workspace_size, fa_get_device_error, fa_strerror,
    fa_bwd_preprocess, fa_bwd_main, fa_bwd_dq_convert,
    fa_bwd_noalloc, FA_BWD_NOALLOC_MAX_WORKSPACE_BYTES, fa_selftest_wait_timeout,
    fa_fwd_decode, fa_decode_workspace_size, fa_decode_split_plan,
    fa_lse_merge, fa_bwd_main_accumulate, fa_convert_f32_bf16, fa_fwd_qk8, fa_fwd_fp8,
    fa_fwd_bias, fa_bwd_bias,
    attention_forward, attention_backward, attention_decode, attention_forward_qk8,
    attention_forward_fp8,
    attention_forward_bias, attention_backward_bias,
)
