"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and the bench.

This module only draws random numbers and names shapes. It holds none of the
attention or RoPE arithmetic, so that neither side of a parity check depends on
the other through it.

Recipe (every workload): a CPU ``torch.Generator`` seeded with ``seed`` draws
iid N(0, 1) fp32 values with ``torch.randn`` in the order q, k, v (decode: q,
k_cache, v_cache), each in contiguous BHSD layout ``[batch, heads, seq, head_dim]``,
and rounds them to bf16 (round-to-nearest-even).  The decode cache is taken to be
already RoPE-rotated: a rotation of iid Gaussian pairs is again iid Gaussian, so
the draw has the distribution of a rotated cache.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, RoPE base and masking."""

    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    D: int
    rope_base: float
    causal: bool = True
    pos_offset: int = 0
    decode_pos: int | None = None  # set for the decode workloads (Sq == 1)

    @property
    def is_decode(self) -> bool:
        return self.decode_pos is not None

    @property
    def keys_attended(self) -> int:
        """Decode: number of cache rows the query at ``decode_pos`` attends."""
        return min(self.Sk, self.decode_pos + 1) if self.is_decode else self.Sk

    def flops(self) -> int:
        """Algorithmic FLOPs (QK^T and PV, 2 FLOPs per multiply-add).

        Causal prefill at Sq == Sk uses the stated convention 2*B*Hq*S^2*D (half of
        the unmasked 4*B*Hq*S^2*D); Sq < Sk counts the allowed (query, key) pairs
        of the bottom-right mask; decode counts 4*B*Hq*L*D over the L keys."""
        if self.is_decode:
            return 4 * self.B * self.Hq * self.keys_attended * self.D
        if not self.causal:
            return 4 * self.B * self.Hq * self.Sq * self.Sk * self.D
        if self.Sq == self.Sk:
            return 2 * self.B * self.Hq * self.Sq * self.Sq * self.D
        off = self.Sk - self.Sq  # row i sees i + off + 1 keys
        pairs = self.Sq * (self.Sq + 1) // 2 + self.Sq * off
        return 4 * self.B * self.Hq * self.D * pairs

    def io_bytes(self) -> int:
        """Algorithmic HBM bytes (bf16): read q, k, v once and write out once.

        Decode reads only the L attended cache rows of K and V."""
        if self.is_decode:
            kv = 2 * self.B * self.Hkv * self.keys_attended * self.D * 2
            return kv + 2 * self.B * self.Hq * self.D * 2
        return 2 * (2 * self.B * self.Hq * self.Sq * self.D + 2 * self.B * self.Hkv * self.Sk * self.D)

    def as_dict(self) -> dict:
        return asdict(self)


# The five workloads: shapes and bases as stated for the method's headline runs.
TINY = Workload("tiny causal MHA", B=1, Hq=2, Hkv=2, Sq=128, Sk=128, D=64, rope_base=10000.0)
SMALL = Workload("small causal MHA", B=2, Hq=8, Hkv=8, Sq=1024, Sk=1024, D=64, rope_base=10000.0)
LLAMA = Workload("Llama-style GQA prefill", B=4, Hq=32, Hkv=8, Sq=4096, Sk=4096, D=128,
                 rope_base=500000.0)
LONG = Workload("long-context GQA prefill", B=1, Hq=64, Hkv=8, Sq=32768, Sk=32768, D=128,
                rope_base=500000.0)
DECODE = Workload("GQA decode over KV cache", B=32, Hq=64, Hkv=8, Sq=1, Sk=8192, D=128,
                  rope_base=500000.0, decode_pos=8191)

CONFIGS = {"tiny": TINY, "small": SMALL, "llama": LLAMA, "long": LONG, "decode": DECODE}


def randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """iid N(0,1) drawn in fp32 on the CPU, rounded to bf16 (RNE)."""
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(w: Workload, seed: int = 0):
    """Return CPU bf16 tensors (q, k, v) for workload ``w``.

    Prefill: q [B,Hq,Sq,D], k and v [B,Hkv,Sk,D].
    Decode:  q [B,Hq,1,D], k_cache (pre-rotated) and v_cache [B,Hkv,Sk,D].
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    q = randn_bf16((w.B, w.Hq, w.Sq, w.D), gen)
    k = randn_bf16((w.B, w.Hkv, w.Sk, w.D), gen)
    v = randn_bf16((w.B, w.Hkv, w.Sk, w.D), gen)
    return q, k, v


def to_f64(t: torch.Tensor):
    """Exact widening of a bf16 tensor to a float64 numpy array."""
    return t.to(torch.float64).numpy()


def plant_spikes(q: torch.Tensor, k: torch.Tensor, row_vals, key_pos, key_vals,
                 key_pos0: int = 0) -> None:
    """Overwrite the last two features of q and k in place (bf16 CPU tensors).

    Query row i of every head gets (row_vals[i % len(row_vals)], 0); key row j of every head
    gets (key_vals[n], 0) where key_pos0 + j == key_pos[n], and (0, 0) elsewhere. The other
    features keep their N(0, 1) draw. Only values are written here: the caller chooses them.
    """
    D = q.shape[-1]
    rv = torch.tensor([float(x) for x in row_vals], dtype=torch.float32)
    idx = torch.arange(q.shape[2]) % len(row_vals)
    q[..., D - 2] = rv[idx].to(q.dtype)
    q[..., D - 1] = 0
    k[..., D - 2:] = 0
    for p, c in zip(key_pos, key_vals):
        j = int(p) - key_pos0
        if 0 <= j < k.shape[2]:
            k[:, :, j, D - 2] = float(c)
