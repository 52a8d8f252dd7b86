"""Exact tiled attention with online softmax for B200 (sm_100a).

The compute lives in libfattn.so (C ABI in include/fattn.h); this package is its thin
Python binding plus the seeded synthetic workload generator used by tests and bench.
"""

from .attention import (  # noqa: F401
    FlashAttnFunction,
    FlashAttnVarlenFunction,
    bwd,
    bwd_noalloc,
    bwd_workspace,
    device_status,
    flash_attn_func,
    flash_attn_varlen_func,
    fwd,
    varlen_bwd,
    varlen_bwd_workspace,
    varlen_fwd,
)
