"""Ring attention over the ranks of a torch.distributed process group.

"Building Self-Attention and Transformer Engines" (codingpancake.com), §6.6 "Ring Attention":
each GPU holds a slice of one sequence's queries, keys and values. It attends its queries to
the key/value block it holds while passing that block to the next GPU of the ring, so after
P steps every query slice has met every block. The per-block results combine exactly through
their log-sum-exp; `rope_attn_fwd_partial` merges each block into the running result.

Slices are contiguous and of equal length L: rank r holds positions r*L .. r*L + L - 1.
Rank r attends its own block first, then the blocks of ranks r-1, r-2, ... as they arrive
from its predecessor. Under the causal mask, the blocks of ranks after r lie wholly in the
future of rank r's queries and are skipped. Their transfer still happens: the ring passes
every block on.

This module is host orchestration only:
* every arithmetic step runs in the library's kernels: `rope_attn_rotate` for the local keys,
  `rope_attn_fwd_partial` per block;
* the transfers are torch.distributed point-to-point operations (NCCL over NVLink between
  GPUs). Each step's send and receive start before the step's kernel and are awaited after
  it, so they overlap with the computation.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib


def ring_steps(rank: int, world: int, causal: bool):
    """The (step, source rank, attended) schedule of one rank: at step t it holds the block
    of rank (rank - t) mod world; under the causal mask blocks of later ranks are skipped."""
    out = []
    for t in range(world):
        src = (rank - t) % world
        out.append((t, src, not (causal and src > rank)))
    return out


def zigzag_step0_fused(c: int, Hq: int, Hkv: int) -> bool:
    """Whether step 0 can attend both query chunks in one masked launch: the kernel's work
    units must not straddle the chunk edge (c a multiple of 128 rows, of 256 when two query
    tiles share a unit, which an odd group size makes them do)."""
    return c % (256 if (Hq // Hkv) % 2 else 128) == 0


def zigzag_calls(rank: int, world: int, causal: bool, fused: bool = True):
    """The kernel calls of one rank under the zig-zag split.

    The sequence is cut into 2*world chunks of c tokens; rank r holds chunk r then chunk
    2*world-1-r in one [.., 2c, ..] tensor ("lo" and "hi" halves). At step t it holds the
    keys/values of rank src = (rank - t) mod world in the same layout. Returns, in order,
    (step, src, query half, key half, masked) with halves "lo", "hi" or "all":
    * step 0: both query chunks against the low key chunk in one masked launch (the low
      chunk's diagonal block; the high chunk is wholly past it, its rows at their own
      positions), then the high diagonal block (masked). With ``fused`` false (chunks that
      do not fall on the kernel's unit edges, see zigzag_step0_fused) the first launch is
      split into the low diagonal block and the wholly past high-on-low block;
    * src < rank: both query chunks against the low key chunk (wholly past: one launch, the
      two query chunks at their own positions);
    * src > rank: the high query chunk against both key chunks (wholly past: one launch);
    * blocks wholly in the future are skipped. Without the mask every step is one launch of
      all queries against all keys.
    Every rank attends 2*world chunk blocks (counting a diagonal one as half) in world + 1
    launches under the mask (world + 2 unfused)."""
    calls = []
    for t in range(world):
        src = (rank - t) % world
        if not causal:
            calls.append((t, src, "all", "all", False))
        elif t == 0 and fused:
            calls += [(0, rank, "all", "lo", True), (0, rank, "hi", "hi", True)]
        elif t == 0:
            calls += [(0, rank, "lo", "lo", True), (0, rank, "hi", "lo", False),
                      (0, rank, "hi", "hi", True)]
        elif src < rank:
            calls.append((t, src, "all", "lo", False))
        else:
            calls.append((t, src, "hi", "all", False))
    return calls


def _zigzag_issue(partial_fn, calls, i, rank, world, c, q, k_cur, v_cur, acc_o, acc_l, out,
                  rope_base, chained=False):
    """Launch call i of zigzag_calls on the views it names. ``chained``: its inputs were
    complete before the previous kernel on the stream started (see rope_attn_fwd_partial)."""
    t, src, qh, kh, masked = calls[i]
    sl = {"lo": slice(0, c), "hi": slice(c, 2 * c), "all": slice(0, 2 * c)}

    def pos(owner, half):
        return (owner if half == "lo" else 2 * world - 1 - owner) * c

    halves = ("lo", "hi") if qh == "all" else (qh,)
    # the first call that writes a query half overwrites its accumulator rows; one call can
    # only overwrite or merge all the rows it covers, so its halves must agree
    written = {h: any(calls[j][2] in (h, "all") for j in range(i)) for h in halves}
    if len(set(written.values())) != 1:
        raise RuntimeError(f"zig-zag call {i} covers a written and an unwritten query half")
    # bf16 rows are written by a half's final call; an "all" call that is final for the low
    # half also writes the high half's rows, which that half's final call overwrites later
    last = any(not any(calls[j][2] in (h, "all") for j in range(i + 1, len(calls)))
               for h in halves)
    q_pos0 = pos(rank, "hi" if qh == "hi" else "lo")
    split, q_pos1 = (c, pos(rank, "hi")) if qh == "all" else (0, 0)
    k_pos0 = pos(src, "hi" if kh == "hi" else "lo")
    partial_fn(q[:, :, sl[qh]], k_cur[:, :, sl[kh]], v_cur[:, :, sl[kh]], acc_o[:, :, sl[qh]],
               acc_l[:, :, sl[qh]], rope_base, q_pos0, k_pos0, causal=masked,
               accumulate=all(written.values()), out=out[:, :, sl[qh]] if last else None,
               q_split=split, q_pos1=q_pos1, **({"chained": True} if chained else {}))


def ring_attention(q, k, v, rope_base: float, causal: bool = True, group=None, out=None, *,
                   layout: str = "contiguous", partial_fn=None, rotate_fn=None):
    """Exact attention of this rank's query slice over the whole ring's keys and values.

    q [B, Hq, L, D], k, v [B, Hkv, L, D]: this rank's slice (positions rank*L ..), keys not
    rotated. Returns out [B, Hq, L, D] (bf16 through the library), this slice of the
    attention over the full sequence. Every rank of the group calls it with the same shapes.
    ``layout="zigzag"`` balances the causal work: the sequence is cut into 2*world chunks of
    c tokens and rank r holds chunk r followed by chunk 2*world-1-r, so q, k, v (and out)
    are [B, H, 2c, D] tensors in that order (see zigzag_calls).
    ``partial_fn`` / ``rotate_fn`` replace the library calls (same signatures as
    `rope_attn_fwd_partial` / `rope_attn_rotate`); the multi-process tests on CPU use them.
    """
    partial_fn = partial_fn or _lib.rope_attn_fwd_partial
    rotate_fn = rotate_fn or _lib.rope_attn_rotate
    # k and v are sent whole to the next rank, and the received blocks must have v's layout
    for name, t in (("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [B, Hkv, L, D] tensor: the ring "
                             f"sends it whole to the next rank")
    distributed = dist.is_available() and dist.is_initialized()
    world = dist.get_world_size(group) if distributed else 1
    rank = dist.get_rank(group) if distributed else 0
    if layout == "zigzag":
        return _ring_zigzag(q, k, v, rope_base, causal, group, out, world, rank, partial_fn,
                            rotate_fn)
    if layout != "contiguous":
        raise ValueError("layout is 'contiguous' or 'zigzag'")
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, L, D]")
    B, Hq, L, D = q.shape
    if k.shape[0] != B or k.shape[2:] != (L, D) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, L, D] with q's B, L and D")

    def peer(r):
        return r if group is None else dist.get_global_rank(group, r)

    # own block (keys rotated here, values as given; read only) and two receive buffers that
    # alternate: the block arriving at step t is attended at step t + 1, while the next one
    # arrives in the other buffer
    own = (torch.empty_like(k), v)
    rotate_fn(k, rope_base, rank * L, out=own[0])
    recv = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    o_acc = torch.empty((B, Hq, L, D), dtype=torch.float32, device=q.device)
    lse_acc = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    sched = ring_steps(rank, world, causal)
    last = max(t for t, _, used in sched if used)
    first = True
    nxt, prv = peer((rank + 1) % world), peer((rank - 1) % world)
    for t, src, used in sched:
        cur = own if t == 0 else recv[(t - 1) % 2]
        reqs = []
        if t < world - 1:
            dst = recv[t % 2]
            ops = [dist.P2POp(dist.isend, cur[0], nxt, group),
                   dist.P2POp(dist.isend, cur[1], nxt, group),
                   dist.P2POp(dist.irecv, dst[0], prv, group),
                   dist.P2POp(dist.irecv, dst[1], prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        if used:
            partial_fn(q, cur[0], cur[1], o_acc, lse_acc, rope_base, rank * L, src * L,
                       causal=causal, accumulate=not first, out=out if t == last else None)
            first = False
        for r in reqs:
            r.wait()
    return out


def _ring_zigzag(q, k, v, rope_base, causal, group, out, world, rank, partial_fn, rotate_fn):
    """ring_attention with the zig-zag split: q, k, v, out are [B, H, 2c, D], chunk rank then
    chunk 2*world-1-rank."""
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("q [B, Hq, 2c, D], k and v [B, Hkv, 2c, D]")
    B, Hq, L, D = q.shape
    if L % 2 or k.shape[0] != B or k.shape[2:] != (L, D):
        raise ValueError("the zig-zag layout needs an even local length shared by q, k, v")
    c = L // 2

    def peer(r):
        return r if group is None else dist.get_global_rank(group, r)

    # own keys rotated at their two chunks' positions, values as given (read only)
    own = (torch.empty_like(k), v)
    rotate_fn(k[:, :, :c], rope_base, rank * c, out=own[0][:, :, :c])
    rotate_fn(k[:, :, c:], rope_base, (2 * world - 1 - rank) * c, out=own[0][:, :, c:])
    recv = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    acc_o = torch.empty((B, Hq, L, D), dtype=torch.float32, device=q.device)
    acc_l = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    calls = zigzag_calls(rank, world, causal, zigzag_step0_fused(c, Hq, k.shape[1]))
    nxt, prv = peer((rank + 1) % world), peer((rank - 1) % world)
    i = 0
    for t in range(world):
        cur = own if t == 0 else recv[(t - 1) % 2]
        reqs = []
        if t < world - 1:
            dst = recv[t % 2]
            ops = [dist.P2POp(dist.isend, cur[0], nxt, group),
                   dist.P2POp(dist.isend, cur[1], nxt, group),
                   dist.P2POp(dist.irecv, dst[0], prv, group),
                   dist.P2POp(dist.irecv, dst[1], prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        first_of_step = True
        while i < len(calls) and calls[i][0] == t:
            # a later call of the same step follows an attention launch whose inputs (and its
            # own) were ready before it; the first call of a step follows the key rotation or
            # the wait for the received block
            _zigzag_issue(partial_fn, calls, i, rank, world, c, q, cur[0], cur[1], acc_o, acc_l,
                          out, rope_base, chained=not first_of_step)
            first_of_step = False
            i += 1
        for r in reqs:
            r.wait()
    return out


def ring_attention_local(q, k, v, rope_base: float, n_ranks: int, causal: bool = True,
                         out=None, on_rank=None, layout: str = "contiguous"):
    """The ring's arithmetic for ``n_ranks`` equal slices of one sequence, every rank's
    schedule run in turn on this device (no process group, no transfers). The kernel calls
    and their order are those of `ring_attention` on each rank, so the output equals the
    distributed result. Use it to validate or time the decomposition on one GPU.

    q [B, Hq, S, D], k, v [B, Hkv, S, D] with S a multiple of n_ranks (of 2*n_ranks for
    ``layout="zigzag"``, where rank r holds chunks r and 2*n_ranks-1-r). ``on_rank(r, phase)``,
    if given, is called with phase "start" before rank r's calls are enqueued and "end"
    after them (for example to record CUDA events). Returns out [B, Hq, S, D] bf16.
    """
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("q [B, Hq, S, D], k and v [B, Hkv, S, D]")
    B, Hq, S, D = q.shape
    if layout == "zigzag":
        return _ring_zigzag_local(q, k, v, rope_base, n_ranks, causal, out, on_rank)
    if layout != "contiguous":
        raise ValueError("layout is 'contiguous' or 'zigzag'")
    if S % n_ranks:
        raise ValueError("the sequence length must be a multiple of n_ranks")
    L = S // n_ranks
    # preparation: the slices, and each rank's keys rotated at its own positions (as the
    # owning rank does before the ring starts)
    qs = [q[:, :, r * L:(r + 1) * L].contiguous() for r in range(n_ranks)]
    blocks = [(_lib.rope_attn_rotate(k[:, :, s * L:(s + 1) * L].contiguous(), rope_base, s * L),
               v[:, :, s * L:(s + 1) * L].contiguous()) for s in range(n_ranks)]
    outs = [torch.empty_like(qs[r]) for r in range(n_ranks)]
    o_acc = torch.empty((B, Hq, L, D), dtype=torch.float32, device=q.device)
    lse_acc = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    # the ring's attention: each rank's blocks in its ring order, merged into its accumulator
    for r in range(n_ranks):
        if on_rank:
            on_rank(r, "start")
        used = [(t, src) for t, src, u in ring_steps(r, n_ranks, causal) if u]
        for i, (_, src) in enumerate(used):
            # every block after the very first follows an attention launch, and all keys were
            # rotated before the first: it may run alongside its predecessor's last wave
            _lib.rope_attn_fwd_partial(qs[r], blocks[src][0], blocks[src][1], o_acc, lse_acc,
                                       rope_base, r * L, src * L, causal=causal,
                                       accumulate=i > 0,
                                       out=outs[r] if i == len(used) - 1 else None,
                                       chained=r > 0 or i > 0)
        if on_rank:
            on_rank(r, "end")
    return torch.cat(outs, dim=2, out=out) if out is not None else torch.cat(outs, dim=2)


def _ring_zigzag_local(q, k, v, rope_base, n, causal, out, on_rank):
    """ring_attention_local with the zig-zag split: each rank's [B, H, 2c, D] tensors are
    assembled first (chunk r, chunk 2n-1-r; keys rotated at their positions), then every
    rank's zigzag_calls run in turn on the other ranks' prepared keys and values."""
    B, Hq, S, D = q.shape
    if S % (2 * n):
        raise ValueError("the zig-zag split needs the sequence length a multiple of 2*n_ranks")
    c = S // (2 * n)

    def rows(chunk):
        return slice(chunk * c, (chunk + 1) * c)

    mine = [(r, 2 * n - 1 - r) for r in range(n)]
    qs = [torch.cat([q[:, :, rows(a)], q[:, :, rows(b)]], dim=2) for a, b in mine]
    vs = [torch.cat([v[:, :, rows(a)], v[:, :, rows(b)]], dim=2) for a, b in mine]
    ks = []
    for a, b in mine:
        kr = torch.empty((B, k.shape[1], 2 * c, D), dtype=k.dtype, device=k.device)
        _lib.rope_attn_rotate(k[:, :, rows(a)], rope_base, a * c, out=kr[:, :, :c])
        _lib.rope_attn_rotate(k[:, :, rows(b)], rope_base, b * c, out=kr[:, :, c:])
        ks.append(kr)
    outs = [torch.empty_like(x) for x in qs]
    acc_o = torch.empty((B, Hq, 2 * c, D), dtype=torch.float32, device=q.device)
    acc_l = torch.empty((B, Hq, 2 * c), dtype=torch.float32, device=q.device)
    for r in range(n):
        if on_rank:
            on_rank(r, "start")
        calls = zigzag_calls(r, n, causal, zigzag_step0_fused(c, Hq, k.shape[1]))
        for i, (_, src, _, _, _) in enumerate(calls):
            # all keys were rotated before the first call (see ring_attention_local)
            _zigzag_issue(_lib.rope_attn_fwd_partial, calls, i, r, n, c, qs[r], ks[src], vs[src],
                          acc_o, acc_l, outs[r], rope_base, chained=r > 0 or i > 0)
        if on_rank:
            on_rank(r, "end")
    if out is None:
        out = torch.empty_like(q)
    for r, (a, b) in enumerate(mine):
        out[:, :, rows(a)] = outs[r][:, :, :c]
        out[:, :, rows(b)] = outs[r][:, :, c:]
    return out
