"""libropeattn Python binding: RoPE + grouped-query causal attention on B200 (sm_100a).

    from transformer_attention_04_b200 import rope_attn_fwd, rope_attn_decode, rope_attn_rotate
"""
from ._lib import (  # noqa: F401
    LIB_PATH,
    RA_ERR_CUDA,
    RA_ERR_DEVICE_TIMEOUT,
    RA_ERR_INVALID_ARG,
    RA_ERR_UNSUPPORTED,
    RA_OK,
    RopeAttnError,
    SIGNATURES,
    lib,
    rope_attn_decode,
    rope_attn_decode_auto_splits,
    rope_attn_decode_noalloc,
    rope_attn_decode_paged,
    rope_attn_decode_step,
    rope_attn_fwd,
    rope_attn_fwd_partial,
    rope_attn_get_device_status,
    rope_attn_prefill,
    rope_attn_profile_enable,
    rope_attn_profile_pause,
    rope_attn_profile_read,
    rope_attn_rotate,
    rope_attn_set_wait_limit,
    rope_attn_version,
)
from .ring import (ring_attention, ring_attention_local, ring_steps, zigzag_calls,  # noqa: F401,E402
                   zigzag_step0_fused)
