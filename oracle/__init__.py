"""fp64 CPU oracle (test infrastructure only; never on the product path)."""
from .ref import (  # noqa: F401
    rope_inv_freq,
    rope_rotate,
    attention,
    query_positions,
    rope_attn_fwd,
    rope_attn_decode,
)
