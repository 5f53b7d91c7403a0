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


def zigzag_steps(rank: int, world: int, causal: bool):
    """The zig-zag schedule of one rank: the sequence is cut into 2*world equal chunks and
    rank r holds chunks r and 2*world-1-r (its pair). At step t it holds the pair of rank
    src = (rank - t) mod world. Returns the (step, src, query half, key half) of every block
    attended, in order; half 0 is the pair's first chunk, half 1 its second. Under the causal
    mask a key chunk that lies wholly after the query chunk is skipped; the two chunks of a
    pair are mirror images, so every rank attends the same number of chunk blocks."""
    def chunk(owner, half):
        return owner if half == 0 else 2 * world - 1 - owner

    out = []
    for t in range(world):
        src = (rank - t) % world
        for qh in (0, 1):
            for kh in (0, 1):
                if not (causal and chunk(src, kh) > chunk(rank, qh)):
                    out.append((t, src, qh, kh))
    return out


def ring_attention(q, k, v, rope_base: float, causal: bool = True, group=None, out=None, *,
                   layout: str = "contiguous", partial_fn=None, rotate_fn=None):
    """Exact attention of this rank's query slice over the whole ring's keys and values.

    q [B, Hq, L, D], k, v [B, Hkv, L, D]: this rank's slice (positions rank*L ..), keys not
    rotated. Returns out [B, Hq, L, D] (bf16 through the library), this slice of the
    attention over the full sequence. Every rank of the group calls it with the same shapes.
    ``layout="zigzag"`` balances the causal work: the sequence is cut into 2*world chunks of
    c tokens and rank r holds chunks r and 2*world-1-r, so q, k, v (and out, if given) are
    pairs (first chunk, second chunk) of [B, H, c, D] tensors, and a pair is returned.
    ``partial_fn`` / ``rotate_fn`` replace the library calls (same signatures as
    `rope_attn_fwd_partial` / `rope_attn_rotate`); the multi-process tests on CPU use them.
    """
    partial_fn = partial_fn or _lib.rope_attn_fwd_partial
    rotate_fn = rotate_fn or _lib.rope_attn_rotate
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
    """ring_attention with the zig-zag split (see zigzag_steps); q, k, v, out are pairs."""
    if len(q) != 2 or len(k) != 2 or len(v) != 2:
        raise ValueError("the zig-zag layout takes (first chunk, second chunk) pairs")
    B, Hq, c, D = q[0].shape
    for t in (q[1], k[0], k[1], v[0], v[1]):
        if t.dim() != 4 or t.shape[0] != B or t.shape[2:] != (c, D):
            raise ValueError("every chunk must be [B, H, c, D] with the same B, c and D")
    if k[0].shape != k[1].shape or v[0].shape != k[0].shape or q[1].shape != q[0].shape:
        raise ValueError("the two chunks of a pair must have the same shape")

    def peer(r):
        return r if group is None else dist.get_global_rank(group, r)

    def pos(owner, half):
        return (owner if half == 0 else 2 * world - 1 - owner) * c

    own = [torch.empty_like(k[0]), torch.empty_like(k[1]), v[0], v[1]]
    rotate_fn(k[0], rope_base, pos(rank, 0), out=own[0])
    rotate_fn(k[1], rope_base, pos(rank, 1), out=own[1])
    recv = [[torch.empty_like(x) for x in own] for _ in range(min(2, world - 1))]
    acc = [(torch.empty((B, Hq, c, D), dtype=torch.float32, device=q[0].device),
            torch.empty((B, Hq, c), dtype=torch.float32, device=q[0].device)) for _ in range(2)]
    if out is None:
        out = (torch.empty_like(q[0]), torch.empty_like(q[1]))
    sched = zigzag_steps(rank, world, causal)
    last = {qh: max(i for i, x in enumerate(sched) if x[2] == qh) for qh in (0, 1)}
    first = {0: True, 1: True}
    nxt, prv = peer((rank + 1) % world), peer((rank - 1) % world)
    i = 0
    for t in range(world):
        cur = own if t == 0 else recv[(t - 1) % 2]
        reqs = []
        if t < world - 1:
            dst = recv[t % 2]
            ops = [dist.P2POp(dist.isend, x, nxt, group) for x in cur]
            ops += [dist.P2POp(dist.irecv, x, prv, group) for x in dst]
            reqs = dist.batch_isend_irecv(ops)
        src = (rank - t) % world
        while i < len(sched) and sched[i][0] == t:
            _, _, qh, kh = sched[i]
            partial_fn(q[qh], cur[kh], cur[2 + kh], acc[qh][0], acc[qh][1], rope_base,
                       pos(rank, qh), pos(src, kh), causal=causal, accumulate=not first[qh],
                       out=out[qh] if i == last[qh] else None)
            first[qh] = False
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
            _lib.rope_attn_fwd_partial(qs[r], blocks[src][0], blocks[src][1], o_acc, lse_acc,
                                       rope_base, r * L, src * L, causal=causal,
                                       accumulate=i > 0,
                                       out=outs[r] if i == len(used) - 1 else None)
        if on_rank:
            on_rank(r, "end")
    return torch.cat(outs, dim=2, out=out) if out is not None else torch.cat(outs, dim=2)


def _ring_zigzag_local(q, k, v, rope_base, n, causal, out, on_rank):
    """ring_attention_local with the zig-zag split: chunk i of the sequence (c tokens at i*c)
    is one contiguous tensor; rank r's blocks follow zigzag_steps."""
    B, Hq, S, D = q.shape
    if S % (2 * n):
        raise ValueError("the zig-zag split needs the sequence length a multiple of 2*n_ranks")
    c = S // (2 * n)
    qs = [q[:, :, i * c:(i + 1) * c].contiguous() for i in range(2 * n)]
    ks = [_lib.rope_attn_rotate(k[:, :, i * c:(i + 1) * c].contiguous(), rope_base, i * c)
          for i in range(2 * n)]
    vs = [v[:, :, i * c:(i + 1) * c].contiguous() for i in range(2 * n)]
    outs = [torch.empty_like(qs[i]) for i in range(2 * n)]
    acc = [(torch.empty((B, Hq, c, D), dtype=torch.float32, device=q.device),
            torch.empty((B, Hq, c), dtype=torch.float32, device=q.device)) for _ in range(2)]

    def chunk(owner, half):
        return owner if half == 0 else 2 * n - 1 - owner

    for r in range(n):
        if on_rank:
            on_rank(r, "start")
        sched = zigzag_steps(r, n, causal)
        last = {qh: max(i for i, x in enumerate(sched) if x[2] == qh) for qh in (0, 1)}
        first = {0: True, 1: True}
        for i, (_, src, qh, kh) in enumerate(sched):
            qi, ki = chunk(r, qh), chunk(src, kh)
            _lib.rope_attn_fwd_partial(qs[qi], ks[ki], vs[ki], acc[qh][0], acc[qh][1], rope_base,
                                       qi * c, ki * c, causal=causal, accumulate=not first[qh],
                                       out=outs[qi] if i == last[qh] else None)
            first[qh] = False
        if on_rank:
            on_rank(r, "end")
    return torch.cat(outs, dim=2, out=out) if out is not None else torch.cat(outs, dim=2)
