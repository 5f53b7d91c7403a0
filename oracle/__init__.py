"""fp64 CPU oracle (test infrastructure only; never on the product path)."""
from .ref import (  # noqa: F401
    rope_inv_freq,
    rope_rotate,
    attention,
    query_positions,
    rope_attn_fwd,
    rope_attn_decode,
    rope_attn_prefill_cached,
    rope_attn_decode_step,
    gather_pages,
    rope_attn_decode_paged,
    rope_attn_fwd_partial,
    merge_partials,
    ring_shards,
    ring_attention,
    zigzag_chunks,
    ring_attention_zigzag,
)
