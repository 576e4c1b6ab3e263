"""Gated DeltaNet recurrence on B200 (sm_100a): Python binding of libgdn.

The compute path is the CUDA library libgdn.so (C ABI declared in
include/gdn.h).  This module only marshals torch tensors into that ABI:
pointers, sizes and the current CUDA stream.  There is no CPU fallback: if the
library is missing or no GPU is present, the calls raise.
"""
from ._lib import (  # noqa: F401
    GdnError,
    STATUS,
    check_async,
    conv1d_silu,
    conv1d_silu_backward,
    decode_step,
    decode_step_fused,
    decode_step_gated,
    gated_norm,
    gated_norm_backward,
    layer_prefill_host,
    lib,
    lib_path,
    prefill,
    prefill_backward,
    prefill_backward_chunked,
    prefill_gated,
    prefill_noalloc,
    prefill_status,
    prefill_workspace_size,
)
