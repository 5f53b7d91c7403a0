"""The ring-attention driver across real processes on CPU (gloo, world sizes 2 and 3).

The driver's schedule and its point-to-point exchanges run as in a multi-GPU job; the two
library calls it makes (key rotation, one block of attention merged into the running result)
are replaced by fp64 stand-ins built from the oracle, so that the test checks the ring logic
itself: which block each rank holds at each step, which blocks it skips, the positions it
passes, the merge order and the final output. The result must equal the oracle's full
attention over the whole sequence.
"""
import itertools
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, Hq, Hkv, S, D, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal((B, Hq, S, D)), g.standard_normal((B, Hkv, S, D)),
            g.standard_normal((B, Hkv, S, D)))


def _worker(rank, world, port, causal, q_out, layout="contiguous"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle
    from transformer_attention_04_b200.ring import ring_attention

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    calls = []

    def cpu_rotate(x, rope_base, pos_offset, out=None):
        r = oracle.rope_rotate(x.numpy(), pos_offset + np.arange(x.shape[2]), rope_base)
        out.copy_(torch.from_numpy(r))
        return out

    def cpu_partial(q, k_rot, v, o_acc, lse_acc, rope_base, q_pos0, k_pos0, causal=True,
                    accumulate=False, out=None, q_split=0, q_pos1=0, chained=False):
        calls.append((q_pos0, k_pos0, bool(accumulate), out is not None))
        if 0 < q_split < q.shape[2]:
            # two query segments: each row's result depends only on its own position (the
            # mask, if any, compares that position with the keys')
            parts = [oracle.rope_attn_fwd_partial(q[:, :, :q_split].numpy(), k_rot.numpy(),
                                                  v.numpy(), rope_base, q_pos0, k_pos0, causal),
                     oracle.rope_attn_fwd_partial(q[:, :, q_split:].numpy(), k_rot.numpy(),
                                                  v.numpy(), rope_base, q_pos1, k_pos0, causal)]
            o = np.concatenate([parts[0][0], parts[1][0]], axis=2)
            lse = np.concatenate([parts[0][1], parts[1][1]], axis=2)
        else:
            o, lse = oracle.rope_attn_fwd_partial(q.numpy(), k_rot.numpy(), v.numpy(),
                                                  rope_base, q_pos0, k_pos0, causal)
        if accumulate:
            o, lse = oracle.merge_partials(o_acc.double().numpy(), lse_acc.double().numpy(), o,
                                           lse)
        o_acc.copy_(torch.from_numpy(o))
        lse_acc.copy_(torch.from_numpy(lse))
        if out is not None:
            out.copy_(torch.from_numpy(o))
        return out

    B, Hq, Hkv, L, D = 1, 4, 2, 6, 8
    q, k, v = _inputs(B, Hq, Hkv, world * L, D, seed=90)
    if layout == "zigzag":
        c = L // 2
        mine = (rank, 2 * world - 1 - rank)
        local = lambda x: torch.from_numpy(
            np.concatenate([x[:, :, i * c:(i + 1) * c] for i in mine], axis=2))
        res = ring_attention(local(q), local(k), local(v), 1000.0, causal=causal,
                             layout="zigzag", partial_fn=cpu_partial, rotate_fn=cpu_rotate)
        res = np.stack([res[:, :, :c].numpy(), res[:, :, c:].numpy()])
    else:
        sl = slice(rank * L, (rank + 1) * L)
        res = ring_attention(torch.from_numpy(q[:, :, sl].copy()),
                             torch.from_numpy(k[:, :, sl].copy()),
                             torch.from_numpy(v[:, :, sl].copy()), 1000.0, causal=causal,
                             partial_fn=cpu_partial, rotate_fn=cpu_rotate).numpy()
    dist.barrier()
    dist.destroy_process_group()
    q_out.put((rank, res, calls))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_attention_gloo_equals_full(world, causal):
    sys.path.insert(0, ROOT)
    import oracle

    port = _free_port()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, q_out))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q_out.get(timeout=180) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    L = 6
    q, k, v = _inputs(1, 4, 2, world * L, 8, seed=90)
    want = oracle.rope_attn_fwd(q, k, v, 1000.0, 0, causal)
    res = np.concatenate([g[1] for g in got], axis=2)
    np.testing.assert_allclose(res, want, atol=1e-5, rtol=0)
    for rank, _, calls in got:
        # own block first, then the predecessors' blocks; causal skips every later rank
        srcs = [kp // L for _, kp, _, _ in calls]
        expect = [(rank - t) % world for t in range(world)]
        if causal:
            expect = [s for s in expect if s <= rank]
        assert srcs == expect
        assert all(qp == rank * L for qp, _, _, _ in calls)
        assert [acc for _, _, acc, _ in calls] == [False] + [True] * (len(calls) - 1)
        assert [o for _, _, _, o in calls] == [False] * (len(calls) - 1) + [True]


def test_ring_steps_schedule():
    sys.path.insert(0, ROOT)
    from transformer_attention_04_b200.ring import ring_steps
    assert ring_steps(0, 1, True) == [(0, 0, True)]
    assert ring_steps(2, 4, True) == [(0, 2, True), (1, 1, True), (2, 0, True), (3, 3, False)]
    assert [u for _, _, u in ring_steps(0, 4, True)] == [True, False, False, False]
    assert all(u for _, _, u in ring_steps(1, 3, False))
    # every block visits every rank once
    for world in (2, 3, 5):
        for r in range(world):
            assert sorted(s for _, s, _ in ring_steps(r, world, False)) == list(range(world))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_zigzag_ring_attention_gloo_equals_full(world, causal):
    sys.path.insert(0, ROOT)
    import oracle

    port = _free_port()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, q_out, "zigzag"))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted([q_out.get(timeout=180) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    L, c = 6, 3
    q, k, v = _inputs(1, 4, 2, world * L, 8, seed=90)
    want = oracle.rope_attn_fwd(q, k, v, 1000.0, 0, causal)
    n_calls = []
    for rank, res, calls in got:
        for half, chunk in enumerate((rank, 2 * world - 1 - rank)):
            np.testing.assert_allclose(res[half], want[:, :, chunk * c:(chunk + 1) * c],
                                       atol=1e-5, rtol=0)
        n_calls.append(len(calls))
        # the first call of the rank overwrites, the last one writes the output
        assert not calls[0][2] and calls[-1][3]
    # balanced: every rank makes the same launches (world unmasked; masked world + 2 here,
    # since 3-row chunks do not fall on the kernel's 128-row unit edges)
    assert n_calls == [world + 2 if causal else world] * world


def test_zigzag_calls_schedule():
    sys.path.insert(0, ROOT)
    from transformer_attention_04_b200.ring import zigzag_calls, zigzag_step0_fused
    halves = {"lo": ["lo"], "hi": ["hi"], "all": ["lo", "hi"]}
    for world, fused in itertools.product((1, 2, 3, 4, 8), (True, False)):
        chunk = lambda owner, h: owner if h == "lo" else 2 * world - 1 - owner  # noqa: E731
        for r in range(world):
            calls = zigzag_calls(r, world, True, fused)
            assert len(calls) == world + (1 if fused else 2)
            # chunk blocks attended (a diagonal one counts half): 2*world on every rank; a
            # masked call may hold a diagonal block and a wholly past one
            work = sum(0.5 if chunk(r, a) == chunk(s, b) else 1
                       for _, s, qh, kh, _ in calls for a in halves[qh] for b in halves[kh])
            assert work == 2 * world
            # the mask is asked for exactly where a call holds a diagonal block
            for _, s, qh, kh, m in calls:
                assert m == any(chunk(r, a) == chunk(s, b) for a in halves[qh] for b in halves[kh])
            # every (query chunk, key chunk) pair with the key chunk not after the query chunk
            # is attended exactly once
            seen = sorted((chunk(r, a), chunk(s, b)) for _, s, qh, kh, _ in calls
                          for a in halves[qh] for b in halves[kh])
            want = sorted((qc, kc) for qc in (chunk(r, "lo"), chunk(r, "hi"))
                          for kc in range(2 * world) if kc <= qc)
            assert seen == want
            assert len(zigzag_calls(r, world, False, fused)) == world
    # the kernel's units cover 128 query rows, 256 for an odd group size
    assert zigzag_step0_fused(256, 8, 2) and zigzag_step0_fused(2048, 64, 8)
    assert not zigzag_step0_fused(300, 8, 2)
    assert zigzag_step0_fused(256, 6, 2) and not zigzag_step0_fused(128, 6, 2)


def test_ring_drivers_reject_bad_arguments():
    # argument errors are raised on the host before any library call (CPU tensors suffice)
    sys.path.insert(0, ROOT)
    from transformer_attention_04_b200.ring import ring_attention, ring_attention_local
    q = torch.zeros(1, 4, 8, 16)
    k = torch.zeros(1, 2, 8, 16)
    with pytest.raises(ValueError):
        ring_attention(q, k[:, :, :6], k, 1e4)                 # k shorter than q
    with pytest.raises(ValueError):
        ring_attention(q, k, k, 1e4, layout="striped")         # unknown layout
    with pytest.raises(ValueError):
        ring_attention(q[:, :, :7], k[:, :, :7], k[:, :, :7], 1e4, layout="zigzag")  # odd length
    with pytest.raises(ValueError, match="contiguous"):
        ring_attention(q, k, torch.zeros(1, 2, 12, 16)[:, :, :8], 1e4)  # v a slice of a longer v
    with pytest.raises(ValueError, match="contiguous"):
        ring_attention(q, torch.zeros(1, 2, 12, 16)[:, :, 4:], k, 1e4, layout="zigzag")
    with pytest.raises(ValueError):
        ring_attention_local(q, k, k, 1e4, 3)                  # 8 tokens over 3 ranks
    with pytest.raises(ValueError):
        ring_attention_local(q, k, k, 1e4, 3, layout="zigzag")  # 8 tokens over 6 chunks
