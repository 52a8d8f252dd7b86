"""CPU fp64 oracle for exact attention. Test infrastructure only (see attn_ref)."""

from .attn_ref import (  # noqa: F401
    ROW_BLOCK,
    allowed_mask,
    attention_backward,
    attention_backward_bhsd,
    attention_forward,
    attention_forward_bhsd,
    attention_forward_fp8,
    decode_attention,
    e4m3_to_float,
    kv_cache_gather,
    softmax_probs,
    varlen_attention_backward,
    varlen_attention_forward,
)
