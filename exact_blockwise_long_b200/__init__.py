"""B200 (sm_100a) exact blockwise ring attention and blockwise feed-forward.

Thin Python binding over the C ABI of ``libringattn.so`` (include/ringattn.h).
Functions take torch CUDA tensors and only marshal pointers, sizes and the
current CUDA stream; every step of the computation runs in the library's
kernels.  PyTorch is used for device memory and streams only.
"""

from ._lib import RA_BF16, RA_F32, RingAttnError, lib  # noqa: F401
from .api import (  # noqa: F401
    ringattn_fwd,
    ringattn_fwd_gqa,
    ringattn_bwd_gqa,
    ringattn_fwd_step,
    ringattn_merge,
    ringattn_bwd,
    ringattn_bwd_phase,
    ringattn_bwd_noalloc,
    ringattn_bwd_workspace_size,
    ringattn_kernel_plan,
    ringattn_bwd_prepare,
    ringattn_bwd_prepare_size,
    ringattn_bwd_pair,
    ringattn_step_host,
    ringattn_step_host_size,
    ringattn_decode,
    ringattn_decode_workspace_size,
    blockwise_ffn,
    blockwise_ffn_bwd,
    ringattn_accumulate,
    ringattn_cast,
    blockwise_layer_bwd,
    blockwise_layer_bwd_workspace_size,
    blockwise_layer_fwd,
    blockwise_layer_fwd_workspace_size,
    blockwise_layer_saved_size,
    blockwise_ffn_bwd_workspace_size,
    blockwise_ffn_workspace_size,
    ringattn_get_error,
    ringattn_selftest_timeout,
)

__all__ = [
    "ringattn_fwd", "ringattn_fwd_gqa", "ringattn_bwd_gqa", "ringattn_fwd_step", "ringattn_merge", "ringattn_bwd", "ringattn_bwd_phase", "ringattn_bwd_noalloc", "ringattn_bwd_workspace_size",
    "ringattn_kernel_plan", "ringattn_bwd_prepare", "ringattn_bwd_prepare_size", "ringattn_bwd_pair", "ringattn_step_host",
    "ringattn_step_host_size",
    "ringattn_decode", "ringattn_decode_workspace_size", "blockwise_ffn", "blockwise_ffn_bwd", "ringattn_accumulate", "ringattn_cast", "blockwise_layer_fwd", "blockwise_layer_bwd", "blockwise_layer_saved_size",
    "blockwise_layer_fwd_workspace_size", "blockwise_layer_bwd_workspace_size", "blockwise_ffn_bwd_workspace_size", "blockwise_ffn_workspace_size", "ringattn_get_error", "ringattn_selftest_timeout",
    "RA_BF16", "RA_F32", "RingAttnError", "lib",
]
