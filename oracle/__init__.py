"""fp64 CPU oracle for the Gated DeltaNet recurrence (test infrastructure).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path never does; it shares no code with
the CUDA library.  See gdn_oracle.c for what each function computes and the
passages it follows.
"""
from .oracle import (  # noqa: F401
    build,
    conv1d_silu,
    conv1d_silu_backward,
    conv1d_silu_f64,
    decode,
    gated_norm,
    gated_norm_backward,
    log_alpha,
    beta,
    max_threads,
    prefill,
    prefill_backward,
    prefill_backward_chunked,
    prefill_chunked,
    prefill_f64,
)
