"""A CPU model of the prefill kernel's tile loop, used only to show that the spike inputs of
spike_cases.py reach the online-softmax rescale and that the GPU parity tests on them would
catch a mistake there.

The model follows the loop of the kernel on one (batch, head): 128-row query tiles, 128-key
tiles visited in ascending order from the first tile inside the window (or 0) to the last
tile with a visible key, the causal / window / sequence-end mask, and the lazily updated
reference maximum: a row keeps its reference m until a tile's maximum exceeds it by more
than 8 (log2 units of the scaled score), and then rescales its running sum l and output O
by alpha = 2^(m_old - m_new). P = 2^(s - m) is rounded to bf16 before it multiplies V, the
row sum takes the unrounded values, exactly as the kernel does. Arithmetic is float64.

`bugs` plants one mistake at a time:
* "l_alpha":  the running sum is not rescaled (l *= alpha dropped);
* "o_alpha":  the running output is not rescaled (O *= alpha dropped);
* "no_redo":  after a jump the tile keeps the P computed with the old reference.
"""
from __future__ import annotations

import math

import numpy as np
import torch

TILE = 128
THRESHOLD = 8.0


def _bf16(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        x = x.astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()


def model_call(q_rot, k_rot, v, causal: bool, off: int, window: int = 0, bugs=()):
    """One launch on one head: q_rot [Sq, D], k_rot and v [Sk, D] (float64, rotated).

    Query row i sits at key index i + off. Returns (o [Sq, D], lse [Sq] natural log,
    stats) with stats counting, over (row, tile), the rescales of a row that already had a
    reference ("rescale") and those whose speculative P would overflow fp32 ("overflow"),
    split by whether the tile was masked ("*_masked")."""
    Sq, D = q_rot.shape
    Sk = k_rot.shape[0]
    sl2 = math.log2(math.e) / math.sqrt(D)
    o = np.zeros((Sq, v.shape[1]))
    lse = np.full(Sq, -np.inf)
    stats = {"rescale": 0, "overflow": 0, "rescale_masked": 0, "overflow_masked": 0,
             "rows_rescaled": 0, "row_mod4_rescaled": np.zeros(4, dtype=np.int64)}
    for q0 in range(0, Sq, TILE):
        rows = np.arange(q0, min(Sq, q0 + TILE))
        n_kv = (Sk + TILE - 1) // TILE
        if causal:
            n_kv = min(n_kv, (min(Sq - 1, q0 + TILE - 1) + off) // TILE + 1)
        j_lo = max(0, q0 + off - window + 1) // TILE if window > 0 else 0
        m = np.full(rows.size, -np.inf)
        l = np.zeros(rows.size)
        acc = np.zeros((rows.size, v.shape[1]))
        rescaled = np.zeros(rows.size, dtype=bool)
        for j in range(j_lo, n_kv):
            keys = np.arange(j * TILE, min(Sk, (j + 1) * TILE))
            s = (q_rot[rows] @ k_rot[keys].T) * sl2
            allowed = np.ones(s.shape, dtype=bool)
            if causal:
                allowed &= keys[None, :] <= rows[:, None] + off
            if window > 0:
                allowed &= keys[None, :] > rows[:, None] + off - window
            masked_tile = (not allowed.all()) or keys.size < TILE
            s = np.where(allowed, s, -np.inf)
            mt = s.max(axis=1)
            m_new = np.maximum(m, mt)
            upd = m_new > m + THRESHOLD
            had = np.isfinite(m)
            real = upd & had
            with np.errstate(invalid="ignore"):
                over = real & (m_new - m > 128.0)
            stats["rescale"] += int(real.sum())
            stats["overflow"] += int(over.sum())
            if masked_tile:
                stats["rescale_masked"] += int(real.sum())
                stats["overflow_masked"] += int(over.sum())
            rescaled |= real
            with np.errstate(invalid="ignore"):
                alpha = np.where(upd, np.exp2(np.where(had, m - m_new, -np.inf)), 1.0)
            m_old = m.copy()
            m = np.where(upd, m_new, m)
            if "l_alpha" not in bugs:
                l = l * alpha
            if "o_alpha" not in bugs:
                acc = acc * alpha[:, None]
            m_use = np.where(np.isfinite(m), m, 0.0)
            if "no_redo" in bugs:
                m_use = np.where(real, m_old, m_use)
            with np.errstate(over="ignore"):
                p = np.exp2(s - m_use[:, None])
            l = l + p.sum(axis=1)
            acc = acc + _bf16(p) @ v[keys]
        o[rows] = acc / l[:, None]
        with np.errstate(divide="ignore"):
            lse[rows] = (m + np.log2(l)) * math.log(2.0)
        stats["rows_rescaled"] += int(rescaled.sum())
        np.add.at(stats["row_mod4_rescaled"], rows[rescaled] % 4, 1)
    return o, lse, stats


def merge(o_a, lse_a, o_b, lse_b):
    """The LSE merge of two partial results (natural-log LSEs)."""
    mx = np.maximum(lse_a, lse_b)
    with np.errstate(invalid="ignore", over="ignore"):
        ea, eb = np.exp(lse_a - mx), np.exp(lse_b - mx)
        return (ea[:, None] * o_a + eb[:, None] * o_b) / (ea + eb)[:, None], mx + np.log(ea + eb)
