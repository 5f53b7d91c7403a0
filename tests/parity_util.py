"""Shared helpers of the GPU parity tests (comparison against the fp64 oracle)."""
import numpy as np
import torch

# Parity bar for bf16 inputs with fp32 accumulation against the fp64 oracle.
MAX_ABS = 2e-2
REL_RMS = 5e-3


def errors(got, want):
    """(max |got - want|, ||got - want||_2 / ||want||_2) in float64."""
    g = got.float().cpu().double().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    w = np.asarray(want, dtype=np.float64)
    d = g - w
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(w), 1e-300))


def assert_parity(got, want, what=""):
    ma, rr = errors(got, want)
    assert np.all(np.isfinite(got.float().cpu().numpy() if isinstance(got, torch.Tensor) else got)), what
    assert ma <= MAX_ABS and rr <= REL_RMS, f"{what}: max_abs={ma:.3e} rel_rms={rr:.3e}"
    return ma, rr


def sample_rows(S: int, block: int = 64, n_mid: int = 3):
    """Rows checked at full size: the first and last blocks plus n_mid evenly spaced blocks
    (every row of attention is independent, so each checked row is an exact check)."""
    rows = set(range(min(block, S)))
    rows |= set(range(max(0, S - block), S))
    for i in range(1, n_mid + 1):
        start = (S * i) // (n_mid + 1)
        rows |= set(range(start, min(S, start + block // 2)))
    return np.array(sorted(rows), dtype=np.int64)
