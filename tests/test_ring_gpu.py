"""GPU parity of ring attention ("Building Self-Attention and Transformer Engines" §6.6)
against the fp64 oracle, through the C ABI.

* One block (rope_attn_fwd_partial): queries rotated in the kernel at q_pos0 + i against
  keys rotated at k_pos0 + j. The block may be the diagonal one, one wholly in the past, one
  straddling the diagonal, or one without the mask. Ragged shapes, D 64 and 128, odd and even
  group sizes. The fp32 output and the LSE are checked, and so is the optional bf16 copy.
* The in-place merge: a block split into two key ranges, merged in either order, equals the
  whole block.
* The ring on one GPU: every rank's schedule run in turn (no kernel waits on another), so
  the concatenated output must equal full causal (or unmasked) attention. At the
  long-context size this is the 8-rank decomposition that the benchmark times, checked on
  sampled rows.
* The driver at world size 1 (NCCL process group of one rank), and canaries around the
  accumulator.
Bar: O max-abs <= 2e-2 and rel-RMS <= 5e-3; LSE max-abs <= 2e-2. The LSE is a log-sum of
scores computed from bf16-rounded rotated operands; its error is the weighted mean of the
score errors, about 2^-8 at these magnitudes.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import transformer_attention_04_b200 as ra
from parity_util import assert_parity, sample_rows
from synthetic import LONG, make_inputs, to_f64

pytestmark = pytest.mark.gpu

LSE_MAX_ABS = 2e-2


def _ok():
    torch.cuda.synchronize()
    st = ra.rope_attn_get_device_status()
    assert st == ra.RA_OK, ra.lib().rope_attn_last_cuda_error()


def _bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _rotated_keys(k_bf16, pos0, base):
    """Keys rotated by the oracle at pos0 + j and rounded to bf16: the same tensor feeds the
    kernel and (widened) the oracle."""
    k64 = to_f64(k_bf16)
    return torch.from_numpy(oracle.rope_rotate(k64, pos0 + np.arange(k64.shape[2]), base)).to(
        torch.bfloat16)


def _check_lse(got, want, what):
    g = got.double().cpu().numpy()
    assert np.all(np.isfinite(g)), what
    err = float(np.max(np.abs(g - want)))
    assert err <= LSE_MAX_ABS, f"{what}: lse max_abs={err:.3e}"


# (B, Hq, Hkv, Sq, Sk, D, q_pos0, k_pos0, causal)
BLOCKS = [
    (1, 4, 2, 200, 200, 128, 300, 300, True),    # the diagonal block of a ring, at an offset
    (1, 8, 2, 333, 257, 128, 1000, 0, True),     # a block wholly in the past: no mask
    (2, 4, 4, 130, 300, 64, 150, 0, True),       # straddling the diagonal
    (1, 6, 2, 129, 64, 64, 0, 4000, False),      # no mask, keys at later positions
    (1, 2, 1, 1, 1, 128, 0, 0, True),            # one row, one key
    (1, 3, 1, 140, 140, 128, 10, 5, True),       # odd group size: one query tile per CTA
    (1, 16, 2, 512, 384, 128, 384, 0, True),     # several tiles, diagonal ending on a tile edge
]


@pytest.mark.parametrize("shape", BLOCKS)
def test_partial_block(shape):
    B, Hq, Hkv, Sq, Sk, D, qp, kp, causal = shape
    base = 500000.0
    q, k, v = _bf16((B, Hq, Sq, D), 1), _bf16((B, Hkv, Sk, D), 2), _bf16((B, Hkv, Sk, D), 3)
    kr = _rotated_keys(k, kp, base)
    want_o, want_l = oracle.rope_attn_fwd_partial(to_f64(q), to_f64(kr), to_f64(v), base, qp, kp,
                                                  causal)
    o_acc = torch.full((B, Hq, Sq, D), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    out = torch.full((B, Hq, Sq, D), float("nan"), device="cuda", dtype=torch.bfloat16)
    ra.rope_attn_fwd_partial(q.cuda(), kr.cuda(), v.cuda(), o_acc, lse, base, qp, kp, causal,
                             accumulate=False, out=out)
    _ok()
    assert_parity(o_acc, want_o, f"o_acc {shape}")
    assert_parity(out, want_o, f"out {shape}")
    _check_lse(lse, want_l, f"{shape}")


@pytest.mark.parametrize("D,split", [(128, 100), (64, 256), (128, 1)])
def test_partial_merge_of_key_ranges(D, split):
    B, Hq, Hkv, Sq, Sk, qp = 1, 8, 2, 300, 520, 600
    base = 10000.0
    q, k, v = _bf16((B, Hq, Sq, D), 4), _bf16((B, Hkv, Sk, D), 5), _bf16((B, Hkv, Sk, D), 6)
    kr = _rotated_keys(k, 0, base)
    want_o, want_l = oracle.rope_attn_fwd_partial(to_f64(q), to_f64(kr), to_f64(v), base, qp, 0,
                                                  True)
    qg, krg, vg = q.cuda(), kr.cuda(), v.cuda()
    parts = [(krg[:, :, :split].contiguous(), vg[:, :, :split].contiguous(), 0),
             (krg[:, :, split:].contiguous(), vg[:, :, split:].contiguous(), split)]
    for order in (parts, parts[::-1]):
        o_acc = torch.full((B, Hq, Sq, D), float("nan"), device="cuda")
        lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
        out = torch.empty((B, Hq, Sq, D), device="cuda", dtype=torch.bfloat16)
        for i, (kk, vv, k0) in enumerate(order):
            ra.rope_attn_fwd_partial(qg, kk, vv, o_acc, lse, base, qp, k0, True,
                                     accumulate=i > 0, out=out if i == 1 else None)
        _ok()
        assert_parity(o_acc, want_o, "merged o_acc")
        assert_parity(out, want_o, "merged out")
        _check_lse(lse, want_l, "merged lse")


@pytest.mark.parametrize("D", [128, 64])
def test_partial_chained_blocks(D):
    # consecutive blocks whose keys were all rotated before the first call, launched with the
    # chained flag: each may run alongside its predecessor and waits for it only before its
    # merge. The merged result must equal the block over all keys.
    B, Hq, Hkv, Sq, Sk, qp, nb = 2, 16, 4, 1024, 2048, 4096, 4
    base = 500000.0
    q, k, v = _bf16((B, Hq, Sq, D), 31), _bf16((B, Hkv, Sk, D), 32), _bf16((B, Hkv, Sk, D), 33)
    kr = _rotated_keys(k, 0, base)
    want_o, want_l = oracle.rope_attn_fwd_partial(to_f64(q), to_f64(kr), to_f64(v), base, qp, 0,
                                                  True)
    qg, krg, vg = q.cuda(), kr.cuda(), v.cuda()
    L = Sk // nb
    blocks = [(krg[:, :, i * L:(i + 1) * L].contiguous(), vg[:, :, i * L:(i + 1) * L].contiguous())
              for i in range(nb)]
    o_acc = torch.full((B, Hq, Sq, D), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    out = torch.empty((B, Hq, Sq, D), device="cuda", dtype=torch.bfloat16)
    for i, (kk, vv) in enumerate(blocks):
        ra.rope_attn_fwd_partial(qg, kk, vv, o_acc, lse, base, qp, i * L, True,
                                 accumulate=i > 0, out=out if i == nb - 1 else None,
                                 chained=i > 0)
    _ok()
    assert_parity(o_acc, want_o, f"chained o_acc D{D}")
    assert_parity(out, want_o, f"chained out D{D}")
    _check_lse(lse, want_l, f"chained lse D{D}")


def test_partial_merge_into_empty_accumulator_rows():
    # an lse_acc of -inf marks an empty row: merging into it takes the block as it is
    B, Hq, Hkv, S, D = 1, 4, 2, 160, 128
    q, k, v = _bf16((B, Hq, S, D), 7), _bf16((B, Hkv, S, D), 8), _bf16((B, Hkv, S, D), 9)
    kr = _rotated_keys(k, 0, 10000.0)
    want_o, want_l = oracle.rope_attn_fwd_partial(to_f64(q), to_f64(kr), to_f64(v), 10000.0, 0, 0,
                                                  True)
    o_acc = torch.zeros((B, Hq, S, D), device="cuda")
    lse = torch.full((B, Hq, S), float("-inf"), device="cuda")
    ra.rope_attn_fwd_partial(q.cuda(), kr.cuda(), v.cuda(), o_acc, lse, 10000.0, 0, 0, True,
                             accumulate=True)
    _ok()
    assert_parity(o_acc, want_o, "o_acc")
    _check_lse(lse, want_l, "lse")


def _ring_on_one_gpu(q, k, v, base, n, causal):
    return ra.ring_attention_local(q, k, v, base, n, causal)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n", [2, 4])
def test_ring_on_one_gpu_equals_full_attention(n, causal):
    B, Hq, Hkv, S, D, base = 1, 8, 2, 1000, 128, 500000.0
    q, k, v = _bf16((B, Hq, S, D), 10), _bf16((B, Hkv, S, D), 11), _bf16((B, Hkv, S, D), 12)
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), base, 0, causal)
    got = _ring_on_one_gpu(q.cuda(), k.cuda(), v.cuda(), base, n, causal)
    _ok()
    assert_parity(got, want, f"ring n={n} causal={causal}")


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("n", [2, 3])
def test_zigzag_ring_on_one_gpu_equals_full_attention(n, causal):
    B, Hq, Hkv, S, D, base = 1, 8, 2, 1200, 128, 500000.0
    q, k, v = _bf16((B, Hq, S, D), 19), _bf16((B, Hkv, S, D), 20), _bf16((B, Hkv, S, D), 21)
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), base, 0, causal)
    got = ra.ring_attention_local(q.cuda(), k.cuda(), v.cuda(), base, n, causal, layout="zigzag")
    _ok()
    assert_parity(got, want, f"zig-zag ring n={n} causal={causal}")


def test_ring_long_context_eight_ranks_sampled_rows():
    # the 32k-token workload as an 8-rank ring (4096 tokens per rank), the decomposition the
    # benchmark times; every checked row is an exact check of that row
    W = LONG
    q, k, v = make_inputs(W, seed=0)
    got = _ring_on_one_gpu(q.cuda(), k.cuda(), v.cuda(), W.rope_base, 8, True)
    _ok()
    rows = sample_rows(W.Sq, block=32, n_mid=3)
    heads = [0, 17, 63]
    want = oracle.rope_attn_fwd(to_f64(q[:, heads]), to_f64(k[:, [h // 8 for h in heads]]),
                                to_f64(v[:, [h // 8 for h in heads]]), W.rope_base, 0, True,
                                rows=rows)
    assert_parity(got[:, heads][:, :, rows], want, "8-rank ring, long context")
    got = ra.ring_attention_local(q.cuda(), k.cuda(), v.cuda(), W.rope_base, 8, True,
                                  layout="zigzag")
    _ok()
    assert_parity(got[:, heads][:, :, rows], want, "8-rank zig-zag ring, long context")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ring_driver_single_rank():
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        B, Hq, Hkv, S, D, base = 2, 4, 2, 300, 64, 10000.0
        q, k, v = _bf16((B, Hq, S, D), 13), _bf16((B, Hkv, S, D), 14), _bf16((B, Hkv, S, D), 15)
        got = ra.ring_attention(q.cuda(), k.cuda(), v.cuda(), base)
        _ok()
    finally:
        dist.destroy_process_group()
    assert_parity(got, oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), base), "driver")


def test_partial_guards():
    GUARD = 4096
    B, Hq, Hkv, Sq, Sk, D = 1, 4, 2, 333, 200, 128
    q, k, v = _bf16((B, Hq, Sq, D), 16), _bf16((B, Hkv, Sk, D), 17), _bf16((B, Hkv, Sk, D), 18)
    kr = _rotated_keys(k, 0, 10000.0)
    n_o, n_l = B * Hq * Sq * D, B * Hq * Sq
    buf_o = torch.empty(n_o + 2 * GUARD, device="cuda")
    buf_l = torch.empty(n_l + 2 * GUARD, device="cuda")
    for b in (buf_o, buf_l):
        b.view(torch.int32).fill_(0x5A5A5A5A)
    o_acc = buf_o[GUARD:GUARD + n_o].view(B, Hq, Sq, D)
    lse = buf_l[GUARD:GUARD + n_l].view(B, Hq, Sq)
    o_acc.fill_(float("nan"))
    lse.fill_(float("nan"))
    q0, kr0, v0 = q.cuda(), kr.cuda(), v.cuda()
    qc, krc, vc = q0.clone(), kr0.clone(), v0.clone()
    ra.rope_attn_fwd_partial(q0, kr0, v0, o_acc, lse, 10000.0, 500, 0, True)
    _ok()
    for b, n in ((buf_o, n_o), (buf_l, n_l)):
        g = b.view(torch.int32)
        assert bool((g[:GUARD] == 0x5A5A5A5A).all()) and bool((g[GUARD + n:] == 0x5A5A5A5A).all())
    assert not bool(torch.isnan(o_acc).any()) and not bool(torch.isnan(lse).any())
    assert torch.equal(q0, qc) and torch.equal(kr0, krc) and torch.equal(v0, vc)


def test_partial_on_views_of_longer_tensors():
    # q rows [40, 240) of a 400-row tensor, keys rows [100, 400) of a 512-row tensor, the
    # accumulator rows [40, 240) of a 400-row one: each call reads and writes only its rows
    B, Hq, Hkv, D, base = 2, 4, 2, 128, 10000.0
    qa, qb, ka, kb = 40, 240, 100, 400
    q_full = _bf16((B, Hq, 400, D), 22)
    k_full, v_full = _bf16((B, Hkv, 512, D), 23), _bf16((B, Hkv, 512, D), 24)
    kr_full = _rotated_keys(k_full, -ka + 700, base)  # row j rotated at 700 + (j - ka)
    q_pos0, k_pos0 = 900, 700
    want_o, want_l = oracle.rope_attn_fwd_partial(
        to_f64(q_full[:, :, qa:qb]), to_f64(kr_full[:, :, ka:kb]), to_f64(v_full[:, :, ka:kb]),
        base, q_pos0, k_pos0, True)
    qg, krg, vg = q_full.cuda(), kr_full.cuda(), v_full.cuda()
    acc_o = torch.full((B, Hq, 400, D), 7.0, device="cuda")
    acc_l = torch.full((B, Hq, 400), 7.0, device="cuda")
    out = torch.full((B, Hq, 400, D), 7.0, device="cuda", dtype=torch.bfloat16)
    ra.rope_attn_fwd_partial(qg[:, :, qa:qb], krg[:, :, ka:kb], vg[:, :, ka:kb],
                             acc_o[:, :, qa:qb], acc_l[:, :, qa:qb], base, q_pos0, k_pos0, True,
                             out=out[:, :, qa:qb])
    _ok()
    assert_parity(acc_o[:, :, qa:qb], want_o, "o_acc view")
    assert_parity(out[:, :, qa:qb], want_o, "out view")
    _check_lse(acc_l[:, :, qa:qb], want_l, "lse view")
    # rows outside the view are untouched
    for t in (acc_o, acc_l, out.float()):
        assert bool((t[:, :, :qa] == 7.0).all()) and bool((t[:, :, qb:] == 7.0).all())


def test_partial_two_query_segments():
    # rows [0, 256) at positions 3000.., rows [256, 400) at 100.. against keys at 5000..
    # (unmasked: two slices of one sequence in one launch)
    B, Hq, Hkv, Sq, Sk, D, base = 1, 8, 2, 400, 300, 64, 500000.0
    split, p0, p1, kp = 256, 3000, 100, 5000
    q, k, v = _bf16((B, Hq, Sq, D), 25), _bf16((B, Hkv, Sk, D), 26), _bf16((B, Hkv, Sk, D), 27)
    kr = _rotated_keys(k, kp, base)
    a = oracle.rope_attn_fwd_partial(to_f64(q[:, :, :split]), to_f64(kr), to_f64(v), base, p0,
                                     kp, False)
    b = oracle.rope_attn_fwd_partial(to_f64(q[:, :, split:]), to_f64(kr), to_f64(v), base, p1,
                                     kp, False)
    want_o = np.concatenate([a[0], b[0]], axis=2)
    want_l = np.concatenate([a[1], b[1]], axis=2)
    o_acc = torch.empty((B, Hq, Sq, D), device="cuda")
    lse = torch.empty((B, Hq, Sq), device="cuda")
    ra.rope_attn_fwd_partial(q.cuda(), kr.cuda(), v.cuda(), o_acc, lse, base, p0, kp, False,
                             q_split=split, q_pos1=p1)
    _ok()
    assert_parity(o_acc, want_o, "two segments")
    _check_lse(lse, want_l, "two segments")


@pytest.mark.parametrize("D,G,Sq,split,Sk,d0,d1", [
    (128, 4, 512, 256, 256, 0, 1000),  # the zig-zag step 0: a diagonal chunk, a wholly past one
    (64, 4, 512, 256, 256, 0, 1000),
    (128, 3, 640, 256, 300, 40, 100),  # odd group size (256-row units), both segments masked
])
def test_partial_two_query_segments_masked(D, G, Sq, split, Sk, d0, d1):
    # a masked block whose two query segments sit at their own positions (rows [0, split) at
    # kp + d0.., rows [split, Sq) at kp + d1..), merged over an earlier unmasked block of keys
    # before kp; the mask compares each row's own position with the keys'
    B, Hkv, base, kp = 1, 2, 500000.0, 5000
    Hq = G * Hkv
    q, k, v = _bf16((B, Hq, Sq, D), 34), _bf16((B, Hkv, Sk, D), 35), _bf16((B, Hkv, Sk, D), 36)
    k0, v0 = _bf16((B, Hkv, 128, D), 37), _bf16((B, Hkv, 128, D), 38)
    kr, kr0 = _rotated_keys(k, kp, base), _rotated_keys(k0, kp - 128, base)
    p0, p1 = kp + d0, kp + d1

    def block(qs, pos, kk, vv, kpos, causal):
        return oracle.rope_attn_fwd_partial(to_f64(qs), to_f64(kk), to_f64(vv), base, pos, kpos,
                                            causal)

    want = []
    for qs, pos in ((q[:, :, :split], p0), (q[:, :, split:], p1)):
        a = block(qs, pos, kr0, v0, kp - 128, False)
        b = block(qs, pos, kr, v, kp, True)
        want.append(oracle.merge_partials(a[0], a[1], b[0], b[1]))
    want_o = np.concatenate([w[0] for w in want], axis=2)
    want_l = np.concatenate([w[1] for w in want], axis=2)
    o_acc = torch.full((B, Hq, Sq, D), float("nan"), device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), device="cuda")
    out = torch.full((B, Hq, Sq, D), float("nan"), device="cuda", dtype=torch.bfloat16)
    qg = q.cuda()
    ra.rope_attn_fwd_partial(qg, kr0.cuda(), v0.cuda(), o_acc, lse, base, p0, kp - 128, False,
                             q_split=split, q_pos1=p1)
    ra.rope_attn_fwd_partial(qg, kr.cuda(), v.cuda(), o_acc, lse, base, p0, kp, True,
                             accumulate=True, out=out, q_split=split, q_pos1=p1)
    _ok()
    assert_parity(o_acc, want_o, "two masked segments")
    assert_parity(out, want_o, "two masked segments, bf16 copy")
    _check_lse(lse, want_l, "two masked segments")


def test_rotate_in_place():
    # 5 heads: one full group of four heads per work item and a ragged group of one
    x = _bf16((1, 5, 333, 128), 29)
    xg = x.cuda()
    y = ra.rope_attn_rotate(xg, 500000.0, 77)
    ra.rope_attn_rotate(xg, 500000.0, 77, out=xg)
    _ok()
    assert torch.equal(xg, y)
    want = oracle.rope_rotate(to_f64(x), 77 + np.arange(333), 500000.0)
    assert np.max(np.abs(y.double().cpu().numpy() - want)) <= 2 ** -7 * max(1.0, np.max(np.abs(want)))


@pytest.mark.parametrize("D", [24, 40, 96, 120, 256])
def test_rotate_any_row_width(D):
    # D / 8 chunks per row: where that does not divide the rotation block, the threads past a
    # tile's last whole row must leave the next tile's first row alone (in place it would
    # otherwise be rotated twice)
    x = _bf16((2, 3, 301, D), 31)
    xg = x.cuda()
    y = ra.rope_attn_rotate(xg, 10000.0, 5)
    ra.rope_attn_rotate(xg, 10000.0, 5, out=xg)
    _ok()
    assert torch.equal(xg, y)
    want = oracle.rope_rotate(to_f64(x), 5 + np.arange(301), 10000.0)
    assert np.max(np.abs(y.double().cpu().numpy() - want)) <= 2 ** -7 * max(1.0, np.max(np.abs(want)))


def test_rotate_views():
    # rotate rows [30, 130) of one tensor into rows [10, 110) of another at positions 500..
    x = _bf16((2, 3, 160, 64), 28)
    xg = x.cuda()
    out = torch.zeros((2, 3, 200, 64), device="cuda", dtype=torch.bfloat16)
    ra.rope_attn_rotate(xg[:, :, 30:130], 10000.0, 500, out=out[:, :, 10:110])
    _ok()
    want = oracle.rope_rotate(to_f64(x[:, :, 30:130]), 500 + np.arange(100), 10000.0)
    got = out[:, :, 10:110].double().cpu().numpy()
    # one bf16 rounding of values of magnitude up to ~4
    assert np.max(np.abs(got - want)) <= 2 ** -7 * max(1.0, np.max(np.abs(want)))
    assert bool((out[:, :, :10] == 0).all()) and bool((out[:, :, 110:] == 0).all())
