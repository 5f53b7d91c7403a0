"""Inputs whose score rows jump after their first key tile, so that the tiled online softmax
must rescale its running output and sum ("Transformer Architecture & Self-Attention
Mechanics", §4 "The Quadratic Bottleneck & FlashAttention": a tile that raises a row's
maximum rescales everything accumulated so far).

The kernel keeps a stale reference maximum until a row's true maximum exceeds it by more
than 8 (log2 units of the scaled score); iid N(0, 1) inputs never get there after the first
tile. Here the last two features (the lowest-frequency RoPE pair) are overwritten:

* query row i gets (a_i, 0) with a_i = 8, 2, -8, 0 for i % 4 = 0, 1, 2, 3, so the lanes of
  one warp disagree on whether to rescale;
* a few "spike" keys get (c, 0); every other key gets (0, 0).

For a row with a = 8 the spike adds about J = 8 c log2(e) / sqrt(D) to the score (in log2
units); the spikes are placed in later key tiles with J = 14, 54 and 194, i.e. jumps of
about 10, 40 and 140 over the previous maximum. The last one makes the speculative
P = 2^(s - m_old) overflow fp32 (> 2^128), so the tile must be redone. Rows with a = 2 see
a quarter of each jump (the first stays under the threshold), rows with a = -8 see spikes
far below their maximum, rows with a = 0 see none.

With RoPE base 5e5 this pair turns by less than 5e-3 rad over the positions used, so the
rotated spike values stay exact in bf16 and the large scores carry no rounding error beyond
that of ordinary scores.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

from synthetic import plant_spikes, randn_bf16

BASE = 500000.0
ROW_VALS = (8.0, 2.0, -8.0, 0.0)
JUMPS = (14.0, 54.0, 194.0)


def key_value(D: int, jump: float) -> float:
    """bf16-exact key feature c giving a score of about `jump` (log2 units) for a = 8."""
    c = jump * math.sqrt(D) / (ROW_VALS[0] * math.log2(math.e))
    return float(torch.tensor(c).to(torch.bfloat16).float())


@dataclass(frozen=True)
class SpikeCase:
    name: str
    kind: str           # "prefill", "partial" or "chunked"
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    D: int
    causal: bool = True
    window: int = 0
    key_pos: tuple = ()
    jumps: tuple = JUMPS
    # partial: a second block of keys (positions Sk.., all visible) merged with accumulate
    q_pos0: int = 0
    Sk2: int = 0
    key_pos2: tuple = ()
    jumps2: tuple = ()
    # chunked: the first P keys are earlier context already in the cache
    P: int = 0


CASES = [
    SpikeCase("causal_d128", "prefill", 1, 4, 2, 1024, 1024, 128, key_pos=(273, 740, 901)),
    SpikeCase("causal_d64", "prefill", 1, 2, 1, 1024, 1024, 64, key_pos=(273, 740, 901)),
    SpikeCase("noncausal_d128", "prefill", 1, 2, 1, 300, 1000, 128, causal=False,
              key_pos=(300, 700, 990)),
    SpikeCase("window_d64", "prefill", 1, 4, 2, 1024, 1024, 64, window=384,
              key_pos=(700, 830, 901)),
    # queries at 1024..1535: the past block (keys 0..1023), then the diagonal block
    # (keys 1024..1535) merged into the accumulator, each with its own jumps
    SpikeCase("partial_accumulate_d128", "partial", 1, 4, 2, 512, 1024, 128, q_pos0=1024,
              key_pos=(273, 740, 901), Sk2=512, key_pos2=(1224, 1424), jumps2=(60.0, 200.0)),
    # earlier context of 640 tokens in the cache (spikes at 273 and 500), then a chunk of 384
    SpikeCase("chunked_cache_d128", "chunked", 1, 4, 2, 384, 384, 128, P=640,
              key_pos=(273, 500, 901)),
]


def case_inputs(c: SpikeCase, seed: int = 0):
    """(q, k, v) bf16 CPU tensors over the whole key range of the case.

    prefill: q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D].
    partial: q at positions q_pos0.. ; k/v hold keys 0 .. Sk+Sk2-1 (both blocks).
    chunked: q holds the chunk's queries (positions P..P+Sq-1); k/v hold keys 0..P+Sk-1.
    """
    g = torch.Generator().manual_seed(seed)
    n_keys = {"prefill": c.Sk, "partial": c.Sk + c.Sk2, "chunked": c.P + c.Sk}[c.kind]
    q = randn_bf16((c.B, c.Hq, c.Sq, c.D), g)
    k = randn_bf16((c.B, c.Hkv, n_keys, c.D), g)
    v = randn_bf16((c.B, c.Hkv, n_keys, c.D), g)
    pos = list(c.key_pos) + list(c.key_pos2)
    vals = [key_value(c.D, j) for j in list(c.jumps) + list(c.jumps2)]
    plant_spikes(q, k, ROW_VALS, pos, vals)
    return q, k, v


def rotated_keys_bf16(k: torch.Tensor, pos0: int = 0) -> torch.Tensor:
    """Keys rotated by the oracle at pos0 + j and rounded to bf16 (what a cache or a ring
    block holds); the same tensor feeds the kernel and, widened, the oracle."""
    import numpy as np

    import oracle
    k64 = k.to(torch.float64).numpy()
    return torch.from_numpy(oracle.rope_rotate(k64, pos0 + np.arange(k64.shape[2]), BASE)).to(
        torch.bfloat16)


def oracle_expected(c: SpikeCase, q, k, v):
    """(out [B,Hq,Sq,D], lse [B,Hq,Sq] or None) from the fp64 oracle for the case's inputs."""
    import numpy as np

    import oracle
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    if c.kind == "prefill":
        return oracle.rope_attn_fwd(f(q), f(k), f(v), BASE, 0, c.causal, window=c.window), None
    if c.kind == "partial":
        kr = rotated_keys_bf16(k)
        return oracle.rope_attn_fwd_partial(f(q), f(kr), f(v), BASE, c.q_pos0, 0, c.causal)
    kc = torch.zeros(c.B, c.Hkv, c.P + c.Sk, c.D, dtype=torch.bfloat16)
    kc[:, :, :c.P] = rotated_keys_bf16(k[:, :, :c.P])
    vc = torch.zeros_like(kc)
    vc[:, :, :c.P] = v[:, :, :c.P]
    out, _, _ = oracle.rope_attn_prefill_cached(f(q), f(k[:, :, c.P:]), f(v[:, :, c.P:]), f(kc),
                                                f(vc), BASE, c.P, c.causal, window=c.window)
    return out, None
