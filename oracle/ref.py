"""Plain fp64 CPU oracle for RoPE + grouped-query causal scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the CUDA
library; both sides receive the same seeded inputs from ``synthetic``.

Everything is written the slow, obvious way: numpy float64, the full score block
materialised per (batch, head), an explicit -inf mask, a plain row softmax. The
functions follow these passages:

* "Multi-Head Attention & Rotary Position Embeddings (RoPE)" (learnllm.online),
  section "Scaled Dot-Product Attention: The O(S^2) Memory Wall" and its
  ``scaled_dot_product_attention`` code: scores = Q K^T / sqrt(d_k), an upper
  triangle of -inf above the diagonal when causal, softmax over the last axis,
  weights times V.
* "Transformer Architecture & Self-Attention Mechanics" (devthesis.com), §1
  (the row-wise softmax A_ij = exp(q_i.k_j/sqrt d_k) / sum_l exp(q_i.k_l/sqrt d_k))
  and §3 "Rotary Position Embeddings (RoPE)": pairs (q_2i, q_2i+1) rotated by
  R(m theta_i) = [[cos, -sin], [sin, cos]], theta_i = 10000^(-2i/d_k).
* "Transformer internals: attention without the mysticism" (ninaddeshpande.com),
  section "Rotary positional embeddings (RoPE)": the base b of theta_i is a free
  parameter (context extension changes it), and section "The KV cache and the
  memory wall": grouped-query attention shares one key/value head among a group
  of query heads.
* "Building Self-Attention and Transformer Engines" (codingpancake.com), FAQ Q2:
  causal masking sets the upper triangle to -inf before the softmax.

Readings where the pages leave a step open (each also listed in the design notes):

* Head sharing: query head h reads key/value head h // (Hq // Hkv) (contiguous
  groups), Hq a multiple of Hkv.
* Positions are bottom-right aligned: query row i sits at absolute position
  pos_offset + (Sk - Sq) + i, key row j at pos_offset + j, and key j is allowed
  iff its position is not after the query's. At Sq == Sk and pos_offset == 0 this
  is exactly triu(-inf, diagonal=1).
* Pairs are adjacent elements (2i, 2i+1); theta_i = base^(-2i/D), i = 0..D/2-1;
  every one of the D dimensions is rotated.
* Decode: the single query at absolute position ``pos`` attends cache rows
  0..min(Sk, pos+1)-1, which hold keys that were already rotated when written.
* Ring attention ("Building Self-Attention and Transformer Engines", §6.6 "Ring Attention"):
  the page gives each GPU a slice of Q, K and V and passes the K/V blocks around a ring while
  each GPU attends its queries to the block it holds; it does not say how the per-block
  results combine. The reading here: every block yields its own normalised output and the
  natural-log sum of exp(scores) of its allowed keys (the LSE); two results over disjoint key
  sets combine exactly by weighting each with exp(its LSE - the LSE of both), which is the
  same regrouping of the softmax denominator that the online softmax uses. Slices are
  contiguous position ranges; under the causal mask a block whose keys all come after the
  slice's queries contributes nothing and is skipped.
* Sliding window ("Building Self-Attention and Transformer Engines", §6.4 "Sliding Window
  Attention (SWA) in Mistral 7B" and FAQ Q10, which limit every token to a window of W
  positions behind it): a query at position p sees the keys at positions p-W+1 .. p, its own
  included, so W = 1 attends only to itself; W = 0 means no window.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rope_inv_freq",
    "rope_rotate",
    "attention",
    "query_positions",
    "rope_attn_fwd",
    "rope_attn_decode",
    "rope_attn_prefill_cached",
    "rope_attn_decode_step",
    "gather_pages",
    "rope_attn_decode_paged",
    "rope_attn_fwd_partial",
    "merge_partials",
    "ring_shards",
    "ring_attention",
    "zigzag_chunks",
    "ring_attention_zigzag",
]


def rope_inv_freq(D: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/D) for i = 0..D/2-1 (devthesis §3 RoPE; base b per
    ninaddeshpande "Rotary positional embeddings")."""
    if D % 2:
        raise ValueError("RoPE needs an even head dimension")
    i = np.arange(D // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * i / D)


def rope_rotate(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotate every adjacent pair (x_2i, x_2i+1) of the rows of ``x`` by m*theta_i.

    ``x`` has shape [..., S, D]; ``positions`` holds the S absolute positions m.
    Per pair: x'_2i = x_2i cos - x_2i+1 sin, x'_2i+1 = x_2i sin + x_2i+1 cos, the
    matrix R(m theta_i) of devthesis §3 applied to the column (x_2i, x_2i+1).
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    theta = rope_inv_freq(D, base)                                   # [D/2]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]  # [S, D/2]
    c, s = np.cos(ang), np.sin(ang)
    even, odd = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


def query_positions(Sq: int, Sk: int, pos_offset: int) -> np.ndarray:
    """Absolute positions of the Sq query rows (bottom-right aligned with the keys)."""
    return pos_offset + (Sk - Sq) + np.arange(Sq, dtype=np.int64)


def _softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax: subtract the row max, exponentiate, divide by the row sum."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, causal: bool,
              rows: np.ndarray | None = None, row_block: int = 1024,
              window: int = 0) -> np.ndarray:
    """softmax(Q K^T / sqrt(D) + M) V with grouped KV heads, in float64.

    q: [B, Hq, Sq, D]; k, v: [B, Hkv, Sk, D] (no RoPE applied here).
    M is -inf where key j lies after query i under the bottom-right alignment
    (j > i + Sk - Sq), i.e. numpy's triu with offset Sk - Sq + 1; zero elsewhere.
    With ``window`` W > 0, M is also -inf where key j lies W or more before the query
    (j <= i + Sk - Sq - W).
    ``rows`` optionally selects which query rows to compute (each row of attention
    is independent of the others, so a subset is an exact check of those rows).
    The score block is materialised ``row_block`` rows at a time to bound memory.
    Returns float64 [B, Hq, len(rows) or Sq, D].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rows = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    scale = 1.0 / np.sqrt(np.float64(D))
    out = np.empty((B, Hq, rows.size, v.shape[-1]), dtype=np.float64)
    cols = np.arange(Sk)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            for r0 in range(0, rows.size, row_block):
                r = rows[r0:r0 + row_block]
                s = (q[b, h, r] @ k[b, kv].T) * scale            # [R, Sk]
                if causal:
                    s = np.where(cols[None, :] > (r[:, None] + (Sk - Sq)), -np.inf, s)
                if window > 0:
                    s = np.where(cols[None, :] <= (r[:, None] + (Sk - Sq) - window), -np.inf, s)
                out[b, h, r0:r0 + r.size] = _softmax_rows(s) @ v[b, kv]
    return out


def rope_attn_fwd(q, k, v, rope_base: float, pos_offset: int = 0, causal: bool = True,
                  rows=None, window: int = 0) -> np.ndarray:
    """The prefill result: rotate Q and K by their absolute positions, then attend.

    q: [B, Hq, Sq, D]; k, v: [B, Hkv, Sk, D]; inputs are widened to float64 first.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    Sq, Sk = q.shape[2], k.shape[2]
    qpos = query_positions(Sq, Sk, pos_offset)
    kpos = pos_offset + np.arange(Sk, dtype=np.int64)
    if rows is not None:
        # rotating only the selected query rows is the same arithmetic per row
        rows = np.asarray(rows, dtype=np.int64)
        q_sel = np.zeros_like(q)
        q_sel[:, :, rows] = rope_rotate(q[:, :, rows], qpos[rows], rope_base)
        q_rot = q_sel
    else:
        q_rot = rope_rotate(q, qpos, rope_base)
    k_rot = rope_rotate(k, kpos, rope_base)
    return attention(q_rot, k_rot, v, causal, rows=rows, window=window)


def rope_attn_decode(q, k_cache_rot, v_cache, rope_base: float, pos: int,
                     window: int = 0) -> np.ndarray:
    """One decode step: the query at absolute position ``pos`` (rotated here) attends
    the first min(Sk, pos+1) rows of an already-rotated key cache (with a window W > 0,
    only the rows pos-W+1 .. pos of those).

    q: [B, Hq, 1, D]; k_cache_rot, v_cache: [B, Hkv, Sk, D]. Returns [B, Hq, 1, D].
    """
    q = np.asarray(q, dtype=np.float64)
    Sk = k_cache_rot.shape[2]
    L = min(Sk, pos + 1)
    lo = max(0, pos - window + 1) if window > 0 else 0
    q_rot = rope_rotate(q, np.array([pos]), rope_base)
    return attention(q_rot, np.asarray(k_cache_rot)[:, :, lo:L], np.asarray(v_cache)[:, :, lo:L],
                     causal=False)


# ----------------------------------------------------------------- KV-cache flow
#
# "Transformer internals: attention without the mysticism", "The KV cache and the memory
# wall", and "Building Self-Attention and Transformer Engines" §6 (GQA & KV-cache
# optimizations) with §6.2 (PagedAttention: the cache split into fixed 16-token blocks):
# the keys and values of past tokens are kept and every new token reads them. Readings (also in the design notes): cache row j holds the key of absolute position
# j, already rotated to that position; a prefill chunk of Sk new tokens starting at
# position pos_offset is written to rows pos_offset .. pos_offset+Sk-1 and its queries attend
# every cache row up to their own position; a decode step writes its new token at row pos[b]
# and attends rows lo .. pos[b] of its own sequence.


def rope_attn_prefill_cached(q, k_new, v_new, k_cache_rot, v_cache, rope_base: float,
                             pos_offset: int, causal: bool = True, window: int = 0):
    """Chunked prefill into a KV cache. Returns (out, k_cache_rot', v_cache').

    q: [B, Hq, Sq, D]; k_new, v_new: [B, Hkv, Sk, D] (keys not rotated);
    k_cache_rot, v_cache: [B, Hkv, S_cache, D] whose rows 0..pos_offset-1 hold the earlier
    context (keys rotated). The chunk's keys are rotated to positions pos_offset + j and
    stored with the values at rows pos_offset + j; the Sq queries sit at positions
    pos_offset + Sk - Sq + i and attend the T = pos_offset + Sk cache rows under the mask.
    """
    k_new = np.asarray(k_new, dtype=np.float64)
    Sk = k_new.shape[2]
    kc = np.array(k_cache_rot, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    T = pos_offset + Sk
    if T > kc.shape[2]:
        raise ValueError("chunk does not fit the cache")
    kc[:, :, pos_offset:T] = rope_rotate(k_new, pos_offset + np.arange(Sk), rope_base)
    vc[:, :, pos_offset:T] = np.asarray(v_new, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    Sq = q.shape[2]
    q_rot = rope_rotate(q, query_positions(Sq, T, 0), rope_base)
    out = attention(q_rot, kc[:, :, :T], vc[:, :, :T], causal, window=window)
    return out, kc, vc


def rope_attn_decode_step(q, k_new, v_new, k_cache_rot, v_cache, rope_base: float, pos,
                          window: int = 0):
    """One decode step of a batch whose sequences sit at their own positions pos[b].

    q: [B, Hq, 1, D]; k_new, v_new: [B, Hkv, 1, D] (the new token's key, not rotated, and
    value), or None to attend the cache as it is; caches [B, Hkv, S_cache, D].
    The new key is rotated to pos[b] and stored with the value at row pos[b]; the query,
    rotated to pos[b], attends rows lo .. pos[b] (lo = pos[b]-W+1 with a window W, else 0).
    Returns (out [B, Hq, 1, D], k_cache_rot', v_cache').
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.array(k_cache_rot, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    B = q.shape[0]
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        p = int(pos[b])
        if k_new is not None:
            kc[b, :, p] = rope_rotate(np.asarray(k_new, dtype=np.float64)[b, :, 0:1],
                                      np.array([p]), rope_base)[:, 0]
            vc[b, :, p] = np.asarray(v_new, dtype=np.float64)[b, :, 0]
        out[b:b + 1] = rope_attn_decode(q[b:b + 1], kc[b:b + 1], vc[b:b + 1], rope_base, p,
                                        window=window)
    return out, kc, vc


def gather_pages(pool, block_table, b: int, n_rows: int):
    """Rows 0..n_rows-1 of sequence b from a paged pool [num_blocks, Hkv, page, D]:
    row j lives in block block_table[b, j // page] at offset j % page ("Building
    Self-Attention and Transformer Engines" §6.2 PagedAttention: a sequence's cache is a
    list of fixed-size physical blocks). Returns [Hkv, n_rows, D]."""
    pool = np.asarray(pool)
    page = pool.shape[2]
    rows = [pool[int(block_table[b, j // page]), :, j % page] for j in range(n_rows)]
    return np.stack(rows, axis=1) if rows else np.zeros((pool.shape[1], 0, pool.shape[3]))


def rope_attn_decode_paged(q, k_new, v_new, k_pool_rot, v_pool, block_table, rope_base: float,
                           pos, window: int = 0):
    """rope_attn_decode_step over a paged cache. Returns (out, k_pool', v_pool').

    The new token (if given) is written to the pool slot of row pos[b]; then each
    sequence's rows 0..pos[b] are gathered through its block table and attended as in the
    contiguous step.
    """
    kp = np.array(k_pool_rot, dtype=np.float64, copy=True)
    vp = np.array(v_pool, dtype=np.float64, copy=True)
    page = kp.shape[2]
    q = np.asarray(q, dtype=np.float64)
    B = q.shape[0]
    out = np.empty(q.shape, dtype=np.float64)
    for b in range(B):
        p = int(pos[b])
        blk, off = int(block_table[b, p // page]), p % page
        if k_new is not None:
            kp[blk, :, off] = rope_rotate(np.asarray(k_new, dtype=np.float64)[b, :, 0:1],
                                          np.array([p]), rope_base)[:, 0]
            vp[blk, :, off] = np.asarray(v_new, dtype=np.float64)[b, :, 0]
        kc = gather_pages(kp, block_table, b, p + 1)[None]
        vc = gather_pages(vp, block_table, b, p + 1)[None]
        out[b:b + 1] = rope_attn_decode(q[b:b + 1], kc, vc, rope_base, p, window=window)
    return out, kp, vp


def rope_attn_fwd_partial(q, k_rot, v, rope_base: float, q_pos0: int, k_pos0: int,
                          causal: bool = True):
    """One block of ring attention: queries at positions q_pos0 + i (rotated here) against
    keys already rotated at positions k_pos0 + j, with their values.

    Key j is allowed to query row i iff causal is false or k_pos0 + j <= q_pos0 + i.
    Returns (o, lse): o [B, Hq, Sq, D] the softmax-weighted values over this block's allowed
    keys, lse [B, Hq, Sq] = ln sum_j exp(q'_i . k'_j / sqrt(D)) over the same keys. A row with
    no allowed key has o = 0 and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k_rot = np.asarray(k_rot, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k_rot.shape
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    qpos = q_pos0 + np.arange(Sq, dtype=np.int64)
    kpos = k_pos0 + np.arange(Sk, dtype=np.int64)
    q_rot = rope_rotate(q, qpos, rope_base)
    scale = 1.0 / np.sqrt(np.float64(D))
    o = np.zeros((B, Hq, Sq, v.shape[-1]), dtype=np.float64)
    lse = np.full((B, Hq, Sq), -np.inf, dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            s = (q_rot[b, h] @ k_rot[b, kv].T) * scale                   # [Sq, Sk]
            if causal:
                s = np.where(kpos[None, :] > qpos[:, None], -np.inf, s)
            m = np.max(s, axis=-1)                                       # [Sq]
            live = np.isfinite(m)
            e = np.exp(s[live] - m[live, None])
            tot = np.sum(e, axis=-1)
            o[b, h, live] = (e @ v[b, kv]) / tot[:, None]
            lse[b, h, live] = m[live] + np.log(tot)
    return o, lse


def merge_partials(o_a, lse_a, o_b, lse_b):
    """Combine two partial results over disjoint key sets into the result over their union.

    The union's denominator is exp(lse_a) + exp(lse_b), so its LSE is
    L = M + ln(exp(lse_a - M) + exp(lse_b - M)) with M the larger LSE, and its output is
    exp(lse_a - L) o_a + exp(lse_b - L) o_b. Rows where both sides are empty stay empty.
    """
    o_a, o_b = np.asarray(o_a, np.float64), np.asarray(o_b, np.float64)
    lse_a, lse_b = np.asarray(lse_a, np.float64), np.asarray(lse_b, np.float64)
    M = np.maximum(lse_a, lse_b)
    both_empty = ~np.isfinite(M)
    Ms = np.where(both_empty, 0.0, M)
    tot = np.exp(lse_a - Ms) + np.exp(lse_b - Ms)
    L = np.where(both_empty, -np.inf, Ms + np.log(np.where(both_empty, 1.0, tot)))
    Ls = np.where(both_empty, 0.0, L)
    w_a = np.where(both_empty, 0.0, np.exp(lse_a - Ls))
    w_b = np.where(both_empty, 0.0, np.exp(lse_b - Ls))
    return w_a[..., None] * o_a + w_b[..., None] * o_b, L


def ring_shards(S: int, n: int):
    """Contiguous slices of S positions over n ranks (the first S % n slices one longer)."""
    q, r = divmod(S, n)
    bounds = [0]
    for i in range(n):
        bounds.append(bounds[-1] + q + (1 if i < r else 0))
    return [(bounds[i], bounds[i + 1]) for i in range(n)]


def ring_attention(q, k, v, rope_base: float, n_ranks: int, causal: bool = True):
    """Ring attention over n_ranks contiguous slices of one sequence (q, k, v [B, H, S, D],
    positions 0..S-1, Sq == Sk).

    Rank r rotates its own keys at their positions, then visits the K/V blocks in ring
    order: its own (step 0), then the block of rank r-1, r-2, ... as they arrive from its
    predecessor. Each visited block gives a partial result that is merged into the running
    one. Under the causal mask the blocks of ranks after r lie wholly in the future of every
    query of r and are skipped. Returns (o [B, Hq, S, D], lse [B, Hq, S]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S = q.shape[2]
    if k.shape[2] != S:
        raise ValueError("ring attention here splits one sequence: Sq must equal Sk")
    shards = ring_shards(S, n_ranks)
    k_rot = [rope_rotate(k[:, :, a:b], np.arange(a, b), rope_base) for a, b in shards]
    outs, lses = [], []
    for r, (qa, qb) in enumerate(shards):
        o_acc, lse_acc = None, None
        for t in range(n_ranks):
            src = (r - t) % n_ranks
            ka, kb = shards[src]
            if causal and src > r:
                continue
            o_p, lse_p = rope_attn_fwd_partial(q[:, :, qa:qb], k_rot[src], v[:, :, ka:kb],
                                               rope_base, qa, ka, causal)
            if o_acc is None:
                o_acc, lse_acc = o_p, lse_p
            else:
                o_acc, lse_acc = merge_partials(o_acc, lse_acc, o_p, lse_p)
        outs.append(o_acc)
        lses.append(lse_acc)
    return np.concatenate(outs, axis=2), np.concatenate(lses, axis=2)


def zigzag_chunks(S: int, n: int):
    """The two position ranges of each of n ranks when one sequence of S positions is cut into
    2n equal chunks and rank r takes chunks r and 2n-1-r."""
    if S % (2 * n):
        raise ValueError("the zig-zag split needs S divisible by 2 * n_ranks")
    c = S // (2 * n)
    return [((r * c, (r + 1) * c), ((2 * n - 1 - r) * c, (2 * n - r) * c)) for r in range(n)]


def ring_attention_zigzag(q, k, v, rope_base: float, n_ranks: int, causal: bool = True):
    """Ring attention with the zig-zag split: rank r holds chunks r and 2n-1-r of the
    sequence, and the blocks passed around the ring are these chunk pairs.

    At step t rank r holds the pair of rank (r - t) mod n. Each of its two query chunks
    attends each of the pair's two key chunks, except (under the causal mask) a key chunk that
    lies wholly after the query chunk; every partial result is merged into that query chunk's
    running result. Returns (o [B, Hq, S, D], lse [B, Hq, S]) in sequence order.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S = q.shape[2]
    if k.shape[2] != S:
        raise ValueError("ring attention here splits one sequence: Sq must equal Sk")
    chunks = zigzag_chunks(S, n_ranks)
    k_rot = {rng: rope_rotate(k[:, :, rng[0]:rng[1]], np.arange(*rng), rope_base)
             for pair in chunks for rng in pair}
    o = np.zeros(q.shape[:3] + (v.shape[-1],))
    lse = np.full(q.shape[:3], -np.inf)
    for r in range(n_ranks):
        for qa, qb in chunks[r]:
            o_acc, lse_acc = None, None
            for t in range(n_ranks):
                for ka, kb in chunks[(r - t) % n_ranks]:
                    if causal and ka > qa:
                        continue  # the key chunk lies wholly after the query chunk
                    o_p, lse_p = rope_attn_fwd_partial(q[:, :, qa:qb], k_rot[(ka, kb)],
                                                       v[:, :, ka:kb], rope_base, qa, ka, causal)
                    if o_acc is None:
                        o_acc, lse_acc = o_p, lse_p
                    else:
                        o_acc, lse_acc = merge_partials(o_acc, lse_acc, o_p, lse_p)
            o[:, :, qa:qb], lse[:, :, qa:qb] = o_acc, lse_acc
    return o, lse
