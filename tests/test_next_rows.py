"""GPU parity of the sliding window, the KV-cache flow and the paged decode against the fp64
oracle, through the C ABI. Bar as everywhere: max-abs <= 2e-2, relative RMS <= 5e-3.

* Sliding window ("Building Self-Attention and Transformer Engines" §6.4): prefill and
  decode, windows smaller than, equal to and larger than a tile, ragged shapes, W = 1.
* Chunked prefill into a cache and the decode step that appends its token at a per-sequence
  position ("Transformer internals: attention without the mysticism", "The KV cache and the
  memory wall"): results, the rows written and the rows that must stay untouched.
* Paged decode through a block table (§6.2 PagedAttention): a pool scattered over shuffled
  blocks gives the bit-identical result of the contiguous cache.
"""
import numpy as np
import pytest
import torch

import oracle
import transformer_attention_04_b200 as ra
from parity_util import assert_parity, errors, MAX_ABS, REL_RMS
from synthetic import Workload, make_inputs, to_f64

pytestmark = pytest.mark.gpu


def _ok():
    torch.cuda.synchronize()
    st = ra.rope_attn_get_device_status()
    assert st == ra.RA_OK, ra.lib().rope_attn_last_cuda_error()


def _bf16(a, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*a, generator=g).to(torch.bfloat16)


# ----------------------------------------------------------------- sliding window, prefill

# (B, Hq, Hkv, Sq, Sk, D, pos_offset, window)
WINDOWED = [
    (1, 2, 2, 128, 128, 64, 0, 32),
    (2, 8, 2, 1024, 1024, 64, 0, 300),
    (1, 4, 1, 333, 700, 128, 7, 128),
    (1, 4, 2, 257, 257, 128, 0, 129),
    (2, 6, 2, 500, 900, 64, 0, 1000),    # window longer than the context: plain causal
    (1, 2, 1, 640, 640, 128, 0, 64),
]


@pytest.mark.parametrize("shape", WINDOWED)
def test_window_prefill(shape):
    B, Hq, Hkv, Sq, Sk, D, off, W = shape
    q, k, v = _bf16((B, Hq, Sq, D), 1), _bf16((B, Hkv, Sk, D), 2), _bf16((B, Hkv, Sk, D), 3)
    out = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), 10000.0, off, True, window=W)
    _ok()
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), 10000.0, off, True, window=W)
    assert_parity(out, want, str(shape))


def test_window_one_is_own_value():
    # W = 1: every query sees only its own key, so out = V at its position, exactly rounded
    q, k, v = _bf16((1, 4, 300, 128), 4), _bf16((1, 2, 300, 128), 5), _bf16((1, 2, 300, 128), 6)
    out = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), 10000.0, 0, True, window=1)
    _ok()
    want = v.repeat_interleave(2, dim=1)
    assert torch.equal(out.cpu(), want)


def test_window_llama_sampled_rows():
    # the bench's prefill shape with a 1024-token window; rows checked across tile edges
    w = Workload("llama_w", 4, 32, 8, 4096, 4096, 128, 500000.0)
    q, k, v = make_inputs(w, 0)
    out = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), w.rope_base, 0, True, window=1024)
    _ok()
    rows = np.array(list(range(0, 16)) + list(range(1020, 1160)) + list(range(4060, 4096)))
    want = oracle.rope_attn_fwd(to_f64(q[:2]), to_f64(k[:2]), to_f64(v[:2]), w.rope_base,
                                rows=rows, window=1024)
    assert_parity(out[:2, :, torch.from_numpy(rows).cuda()], want, "llama window 1024")


def test_window_covering_context_equals_causal_bitwise():
    q, k, v = _bf16((1, 8, 777, 128), 7), _bf16((1, 2, 777, 128), 8), _bf16((1, 2, 777, 128), 9)
    a = ra.rope_attn_fwd(q.cuda(), k.cuda(), v.cuda(), 10000.0, 0, True)
    b = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), 10000.0, 0, True, window=777)
    _ok()
    assert torch.equal(a, b)


def test_window_argument_errors():
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ra.RopeAttnError):
        ra.rope_attn_prefill(q, q[:, :1], q[:, :1], 10000.0, 0, False, window=8)  # needs causal
    with pytest.raises(ra.RopeAttnError):
        ra.rope_attn_prefill(q, q[:, :1], q[:, :1], 10000.0, 0, True, window=-1)


# ----------------------------------------------------------------- chunked prefill into a cache

def test_prefill_to_cache_equals_plain_prefill():
    B, Hq, Hkv, S, D, cap = 2, 8, 2, 600, 128, 1024
    q, k, v = _bf16((B, Hq, S, D), 10), _bf16((B, Hkv, S, D), 11), _bf16((B, Hkv, S, D), 12)
    kc = torch.full((B, Hkv, cap, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = kc.clone()
    gq, gk, gv = q.cuda(), k.cuda(), v.cuda()
    out = ra.rope_attn_prefill(gq, gk, gv, 500000.0, 0, True, k_cache_rot=kc, v_cache=vc)
    ref = ra.rope_attn_fwd(gq, gk, gv, 500000.0, 0, True)
    krot = ra.rope_attn_rotate(gk, 500000.0, 0)
    _ok()
    assert torch.equal(out, ref)               # same rotated keys, same kernel: same bits
    assert torch.equal(kc[:, :, :S], krot)
    assert torch.equal(vc[:, :, :S], gv)
    assert torch.isnan(kc[:, :, S:].float()).all() and torch.isnan(vc[:, :, S:].float()).all()


@pytest.mark.parametrize("P,Sk,Sq,W", [(300, 200, 200, 0), (1000, 77, 77, 0), (128, 256, 256, 0),
                                        (513, 300, 300, 256), (640, 64, 1, 0)])
def test_chunked_prefill(P, Sk, Sq, W):
    # earlier context of P tokens already in the cache, then a chunk of Sk new tokens
    B, Hq, Hkv, D, cap = 2, 4, 2, 128, 1600
    ctx_k, ctx_v = _bf16((B, Hkv, P, D), 20), _bf16((B, Hkv, P, D), 21)
    q, k, v = _bf16((B, Hq, Sq, D), 22), _bf16((B, Hkv, Sk, D), 23), _bf16((B, Hkv, Sk, D), 24)
    # the earlier rows as a cache would hold them: keys rotated (here by the oracle, in fp64,
    # then rounded to bf16), values as they are; rows past them are garbage (NaN)
    kc_in = torch.full((B, Hkv, cap, D), float("nan"), dtype=torch.bfloat16)
    vc_in = kc_in.clone()
    kc_in[:, :, :P] = torch.from_numpy(oracle.rope_rotate(to_f64(ctx_k), np.arange(P),
                                                          10000.0)).to(torch.bfloat16)
    vc_in[:, :, :P] = ctx_v
    kc, vc = kc_in.cuda(), vc_in.cuda()
    kc0 = kc[:, :, :P].clone()
    out = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), 10000.0, P, True, window=W,
                               k_cache_rot=kc, v_cache=vc)
    _ok()
    want, wk, wv = oracle.rope_attn_prefill_cached(to_f64(q), to_f64(k), to_f64(v), to_f64(kc_in),
                                                   to_f64(vc_in), 10000.0, P, window=W)
    assert_parity(out, want, f"chunk P={P}")
    assert torch.equal(kc[:, :, :P], kc0)                            # earlier rows untouched
    ma, _ = errors(kc[:, :, P:P + Sk], wk[:, :, P:P + Sk])           # new rows: rotated keys
    assert ma <= 2.0 ** -7 * 8                                        # one bf16 ulp at |x| < 8
    assert torch.equal(vc[:, :, P:P + Sk].cpu(), v)
    assert torch.isnan(kc[:, :, P + Sk:].float()).all()              # rows past T untouched


# ----------------------------------------------------------------- decode step with append

def _decode_case(seed, B, Hq, Hkv, cap, D, pos, fill_nan=True):
    q = _bf16((B, Hq, 1, D), seed)
    kn, vn = _bf16((B, Hkv, 1, D), seed + 1), _bf16((B, Hkv, 1, D), seed + 2)
    kc, vc = _bf16((B, Hkv, cap, D), seed + 3), _bf16((B, Hkv, cap, D), seed + 4)
    if fill_nan:  # rows past each sequence's end hold garbage the kernel must never use
        for b, p in enumerate(pos):
            kc[b, :, p + 1:] = float("nan")
            vc[b, :, p + 1:] = float("nan")
    return q, kn, vn, kc, vc


@pytest.mark.parametrize("W", [0, 100, 4096])
def test_decode_step_varlen_append(W):
    B, Hq, Hkv, cap, D = 6, 16, 2, 3000, 128
    pos = [2999, 0, 63, 64, 1500, 2048]
    q, kn, vn, kc, vc = _decode_case(30, B, Hq, Hkv, cap, D, pos)
    gkc, gvc = kc.cuda(), vc.cuda()
    gpos = torch.tensor(pos, dtype=torch.int32, device="cuda")
    out = ra.rope_attn_decode_step(q.cuda(), gkc, gvc, gpos, max(pos), 500000.0, kn.cuda(),
                                   vn.cuda(), window=W)
    _ok()
    want, wk, wv = oracle.rope_attn_decode_step(to_f64(q), to_f64(kn), to_f64(vn), to_f64(kc),
                                                to_f64(vc), 500000.0, pos, W)
    assert_parity(out, want, f"decode step W={W}")
    for b, p in enumerate(pos):
        # the appended row is the library's own rotation of the new key, bit for bit
        rot = ra.rope_attn_rotate(kn[b:b + 1].cuda(), 500000.0, p)
        assert torch.equal(gkc[b, :, p], rot[0, :, 0])
        assert torch.equal(gvc[b, :, p].cpu(), vn[b, :, 0])
        # every other row is untouched (NaN payloads compared as bits)
        keep = [j for j in range(cap) if j != p]
        assert torch.equal(gkc[b, :, keep].cpu().view(torch.int16), kc[b, :, keep].view(torch.int16))


def test_decode_step_without_append_matches_decode():
    # all sequences at the last row, nothing appended: the plain decode entry's result
    B, Hq, Hkv, S, D = 4, 32, 8, 2048, 128
    q, kc, vc = _bf16((B, Hq, 1, D), 40), _bf16((B, Hkv, S, D), 41), _bf16((B, Hkv, S, D), 42)
    gq, gkc, gvc = q.cuda(), kc.cuda(), vc.cuda()
    a = ra.rope_attn_decode(gq, gkc, gvc, 500000.0, S - 1)
    b = ra.rope_attn_decode_step(gq, gkc, gvc, torch.full((B,), S - 1, dtype=torch.int32,
                                                          device="cuda"), S - 1, 500000.0)
    _ok()
    assert torch.equal(a, b)


def test_prefill_then_token_by_token_decode():
    # prompt of 700 tokens prefilled into the cache, then 6 decode steps each appending its
    # own token: every output row equals the same row of one prefill over the 706 tokens
    B, Hq, Hkv, D, cap, P, n = 2, 8, 2, 128, 1024, 700, 6
    q, k, v = _bf16((B, Hq, P + n, D), 50), _bf16((B, Hkv, P + n, D), 51), _bf16((B, Hkv, P + n, D), 52)
    gq, gk, gv = q.cuda(), k.cuda(), v.cuda()
    kc = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = [ra.rope_attn_prefill(gq[:, :, :P].contiguous(), gk[:, :, :P].contiguous(),
                                 gv[:, :, :P].contiguous(), 500000.0, 0, True,
                                 k_cache_rot=kc, v_cache=vc)]
    for t in range(P, P + n):
        pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
        outs.append(ra.rope_attn_decode_step(gq[:, :, t:t + 1].contiguous(), kc, vc, pos, t,
                                             500000.0, gk[:, :, t:t + 1].contiguous(),
                                             gv[:, :, t:t + 1].contiguous()))
    _ok()
    got = torch.cat(outs, dim=2)
    rows = np.array(list(range(0, 8)) + list(range(690, P + n)))
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), 500000.0, rows=rows)
    assert_parity(got[:, :, torch.from_numpy(rows).cuda()], want, "prefill + decode")


def test_decode_step_bad_position_is_reported():
    B, Hq, Hkv, cap, D = 2, 8, 2, 512, 64
    q, kn, vn, kc, vc = _decode_case(60, B, Hq, Hkv, cap, D, [100, 200], fill_nan=False)
    gkc = kc.cuda()
    pos = torch.tensor([100, 300], dtype=torch.int32, device="cuda")  # 300 > max_pos = 200
    ra.rope_attn_decode_step(q.cuda(), gkc, vc.cuda(), pos, 200, 10000.0, kn.cuda(), vn.cuda())
    torch.cuda.synchronize()
    assert ra.rope_attn_get_device_status() == ra.RA_ERR_INVALID_ARG
    assert torch.equal(gkc[1].cpu(), kc[1])  # the refused sequence wrote nothing
    assert ra.rope_attn_get_device_status() == ra.RA_OK  # the status was cleared
    with pytest.raises(ra.RopeAttnError):  # max_pos must lie inside the cache
        ra.rope_attn_decode_step(q.cuda(), gkc, vc.cuda(), pos, cap, 10000.0)


# ----------------------------------------------------------------- paged decode

def _to_pool(kc, vc, page, n_extra, seed):
    """Scatter contiguous caches [B, Hkv, cap, D] over a shuffled pool with n_extra spare
    blocks (filled with NaN), returning pool_k, pool_v, table."""
    B, Hkv, cap, D = kc.shape
    per = cap // page
    nb = B * per + n_extra
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(seed))
    table = perm[: B * per].view(B, per).to(torch.int32)
    pk = torch.full((nb, Hkv, page, D), float("nan"), dtype=torch.bfloat16)
    pv = pk.clone()
    idx = table.view(-1).long()
    pk[idx] = kc.view(B, Hkv, per, page, D).permute(0, 2, 1, 3, 4).reshape(B * per, Hkv, page, D)
    pv[idx] = vc.view(B, Hkv, per, page, D).permute(0, 2, 1, 3, 4).reshape(B * per, Hkv, page, D)
    return pk, pv, table


@pytest.mark.parametrize("page,W", [(16, 0), (16, 300), (64, 0), (8, 40), (32, 0)])
def test_paged_equals_contiguous(page, W):
    B, Hq, Hkv, cap, D = 5, 16, 4, 1024, 128
    pos = [1023, 15, 16, 500, 777]
    q, kn, vn, kc, vc = _decode_case(70, B, Hq, Hkv, cap, D, pos)
    pk, pv, table = _to_pool(kc, vc, page, 7, 71)
    gpos = torch.tensor(pos, dtype=torch.int32, device="cuda")
    gkc, gvc, gpk, gpv = kc.cuda(), vc.cuda(), pk.cuda(), pv.cuda()
    a = ra.rope_attn_decode_step(q.cuda(), gkc, gvc, gpos, max(pos), 500000.0, kn.cuda(),
                                 vn.cuda(), window=W)
    b = ra.rope_attn_decode_paged(q.cuda(), gpk, gpv, table.cuda(), gpos, max(pos), 500000.0,
                                  kn.cuda(), vn.cuda(), window=W)
    _ok()
    assert torch.equal(a, b)  # same rows in the same tiles: the same bits
    want, _, _ = oracle.rope_attn_decode_paged(to_f64(q), to_f64(kn), to_f64(vn), to_f64(pk),
                                               to_f64(pv), table.numpy(), 500000.0, pos, W)
    assert_parity(b, want, f"paged {page} W={W}")
    # the appended rows landed in the right pages
    for bb, p in enumerate(pos):
        blk, off = int(table[bb, p // page]), p % page
        assert torch.equal(gpk[blk, :, off], gkc[bb, :, p])
        assert torch.equal(gpv[blk, :, off], gvc[bb, :, p])


def test_paged_bench_shape_against_oracle_sampled():
    # the decode workload (B32 Hq64 Hkv8, 8192 rows each) in 16-token pages; batches 0 and 31
    B, Hq, Hkv, S, D, page = 32, 64, 8, 8192, 128, 16
    q, kc, vc = make_inputs(Workload("decode", B, Hq, Hkv, 1, S, D, 500000.0), 0)
    pk, pv, table = _to_pool(kc, vc, page, 0, 72)
    pos = torch.full((B,), S - 1, dtype=torch.int32)
    out = ra.rope_attn_decode_paged(q.cuda(), pk.cuda(), pv.cuda(), table.cuda(), pos.cuda(),
                                    S - 1, 500000.0)
    _ok()
    for b in (0, 31):
        want = oracle.rope_attn_decode(to_f64(q[b:b + 1]), to_f64(kc[b:b + 1]),
                                       to_f64(vc[b:b + 1]), 500000.0, S - 1)
        ma, rr = errors(out[b:b + 1], want)
        assert ma <= MAX_ABS and rr <= REL_RMS, (b, ma, rr)


def test_paged_bad_block_is_reported():
    B, Hq, Hkv, cap, D, page = 2, 8, 2, 256, 64, 16
    q, kn, vn, kc, vc = _decode_case(80, B, Hq, Hkv, cap, D, [100, 200], fill_nan=False)
    pk, pv, table = _to_pool(kc, vc, page, 0, 81)
    table[1, 200 // page] = pk.shape[0] + 5  # the page that receives sequence 1's token
    gpk = pk.cuda()
    pos = torch.tensor([100, 200], dtype=torch.int32, device="cuda")
    ra.rope_attn_decode_paged(q.cuda(), gpk, pv.cuda(), table.cuda(), pos, 200, 10000.0,
                              kn.cuda(), vn.cuda())
    torch.cuda.synchronize()
    assert ra.rope_attn_get_device_status() == ra.RA_ERR_INVALID_ARG
    # sequence 0 appended normally; nothing was written for sequence 1
    blk0 = int(table[0, 100 // page])
    assert not torch.equal(gpk[blk0, :, 100 % page].cpu(), pk[blk0, :, 100 % page])
    changed = (gpk.cpu().view(torch.int16) != pk.view(torch.int16)).any(dim=(1, 2, 3))
    assert int(changed.sum()) == 1


# ----------------------------------------------------------------- head dimension 64

@pytest.mark.parametrize("W", [0, 50])
def test_decode_step_and_paged_d64(W):
    B, Hq, Hkv, cap, D, page = 3, 12, 3, 512, 64, 32
    pos = [511, 200, 31]
    q, kn, vn, kc, vc = _decode_case(90, B, Hq, Hkv, cap, D, pos)
    pk, pv, table = _to_pool(kc, vc, page, 3, 91)
    gpos = torch.tensor(pos, dtype=torch.int32, device="cuda")
    a = ra.rope_attn_decode_step(q.cuda(), kc.cuda(), vc.cuda(), gpos, max(pos), 10000.0,
                                 kn.cuda(), vn.cuda(), window=W)
    b = ra.rope_attn_decode_paged(q.cuda(), pk.cuda(), pv.cuda(), table.cuda(), gpos, max(pos),
                                  10000.0, kn.cuda(), vn.cuda(), window=W)
    _ok()
    assert torch.equal(a, b)
    want, _, _ = oracle.rope_attn_decode_step(to_f64(q), to_f64(kn), to_f64(vn), to_f64(kc),
                                              to_f64(vc), 10000.0, pos, W)
    assert_parity(a, want, f"d64 W={W}")


def test_chunked_prefill_d64_non_multiple_of_tile():
    B, Hq, Hkv, D, cap, P, Sk = 1, 6, 2, 64, 700, 250, 333
    ctx_k, ctx_v = _bf16((B, Hkv, P, D), 92), _bf16((B, Hkv, P, D), 93)
    q, k, v = _bf16((B, Hq, Sk, D), 94), _bf16((B, Hkv, Sk, D), 95), _bf16((B, Hkv, Sk, D), 96)
    kc_in = torch.zeros(B, Hkv, cap, D, dtype=torch.bfloat16)
    vc_in = torch.zeros_like(kc_in)
    kc_in[:, :, :P] = torch.from_numpy(oracle.rope_rotate(to_f64(ctx_k), np.arange(P),
                                                          10000.0)).to(torch.bfloat16)
    vc_in[:, :, :P] = ctx_v
    kc, vc = kc_in.cuda(), vc_in.cuda()
    out = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), 10000.0, P, True, window=100,
                               k_cache_rot=kc, v_cache=vc)
    _ok()
    want, _, _ = oracle.rope_attn_prefill_cached(to_f64(q), to_f64(k), to_f64(v), to_f64(kc_in),
                                                 to_f64(vc_in), 10000.0, P, window=100)
    assert_parity(out, want, "chunked d64 window")
