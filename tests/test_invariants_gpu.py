"""GPU properties that need no oracle: what the method fixes for any input.

* V == 1 gives O == 1 (softmax rows sum to one);
* causal row 0 attends only key 0, so O[:, :, 0] == V[0] bit for bit;
* Q == 0 gives the running prefix mean of V;
* grouped-query output equals multi-head output with K/V repeated per group, bit for bit;
* shifting every position (pos_offset) leaves the result unchanged up to rounding;
* decode at position S-1 over a rotate()d cache equals the last prefill row;
* the decode result does not depend on the number of splits;
* a kernel wait that runs out reports RA_ERR_DEVICE_TIMEOUT and leaves the context usable.
"""
import numpy as np
import pytest
import torch

import transformer_attention_04_b200 as ra
from parity_util import MAX_ABS, REL_RMS, errors

pytestmark = pytest.mark.gpu


def rnd(*shape, seed=0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("D", [64, 128])
def test_ones_v_gives_ones(D):
    q, k = rnd(2, 4, 300, D, seed=1), rnd(2, 2, 300, D, seed=2)
    v = torch.ones(2, 2, 300, D, dtype=torch.bfloat16, device="cuda")
    o = ra.rope_attn_fwd(q, k, v, 10000.0)
    # P is rounded to bf16 before P.V while the row sum uses the unrounded values
    assert (o.float() - 1).abs().max().item() <= 8e-3


@pytest.mark.parametrize("D", [64, 128])
def test_causal_row0_is_v0(D):
    q, k, v = rnd(1, 4, 260, D, seed=3), rnd(1, 2, 260, D, seed=4), rnd(1, 2, 260, D, seed=5)
    o = ra.rope_attn_fwd(q, k, v, 10000.0)
    assert torch.equal(o[:, :, 0], v.repeat_interleave(2, dim=1)[:, :, 0])


def test_zero_q_prefix_mean():
    S = 700
    q = torch.zeros(1, 2, S, 128, dtype=torch.bfloat16, device="cuda")
    k, v = rnd(1, 2, S, 128, seed=6), rnd(1, 2, S, 128, seed=7)
    o = ra.rope_attn_fwd(q, k, v, 500000.0)
    pm = v.double().cumsum(2) / torch.arange(1, S + 1, device="cuda").double()[None, None, :, None]
    ma, rr = errors(o, pm.cpu().numpy())
    assert ma <= MAX_ABS and rr <= REL_RMS


@pytest.mark.parametrize("G", [2, 4, 8, 3])
def test_gqa_equals_repeated_mha(G):
    Hkv = 2
    q = rnd(2, Hkv * G, 400, 128, seed=8)
    k, v = rnd(2, Hkv, 400, 128, seed=9), rnd(2, Hkv, 400, 128, seed=10)
    o = ra.rope_attn_fwd(q, k, v, 500000.0)
    o_mha = ra.rope_attn_fwd(q, k.repeat_interleave(G, 1).contiguous(),
                             v.repeat_interleave(G, 1).contiguous(), 500000.0)
    assert torch.equal(o, o_mha)


def test_pos_offset_shift_invariance():
    q, k, v = rnd(1, 4, 500, 128, seed=11), rnd(1, 2, 500, 128, seed=12), rnd(1, 2, 500, 128, seed=13)
    o0 = ra.rope_attn_fwd(q, k, v, 500000.0, pos_offset=0)
    for c in (1, 4097, 100000):
        oc = ra.rope_attn_fwd(q, k, v, 500000.0, pos_offset=c)
        ma, rr = errors(oc, o0.double().cpu().numpy())
        assert ma <= MAX_ABS and rr <= REL_RMS, (c, ma, rr)


def test_decode_equals_last_prefill_row():
    S = 1500
    q, k, v = rnd(2, 16, S, 128, seed=14), rnd(2, 2, S, 128, seed=15), rnd(2, 2, S, 128, seed=16)
    full = ra.rope_attn_fwd(q, k, v, 500000.0)
    k_cache = ra.rope_attn_rotate(k, 500000.0, 0)
    d = ra.rope_attn_decode(q[:, :, S - 1:].contiguous(), k_cache, v, 500000.0, S - 1)
    ma, rr = errors(d[:, :, 0], full[:, :, S - 1].double().cpu().numpy())
    assert ma <= MAX_ABS and rr <= REL_RMS


def test_decode_independent_of_splits():
    q, kc, vc = rnd(4, 16, 1, 128, seed=17), rnd(4, 2, 3000, 128, seed=18), rnd(4, 2, 3000, 128, seed=19)
    ref = ra.rope_attn_decode(q, kc, vc, 500000.0, 2999, n_splits=1)
    for s in (2, 3, 7, 16, 47):
        o = ra.rope_attn_decode(q, kc, vc, 500000.0, 2999, n_splits=s)
        assert (o.float() - ref.float()).abs().max().item() <= 1.6e-2


def test_wait_timeout_reports_and_recovers():
    q, k, v = rnd(1, 4, 1024, 128, seed=20), rnd(1, 2, 1024, 128, seed=21), rnd(1, 2, 1024, 128, seed=22)
    good = ra.rope_attn_fwd(q, k, v, 500000.0)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    old = ra.rope_attn_set_wait_limit(0)
    try:
        ra.rope_attn_fwd(q, k, v, 500000.0)
        st1 = ra.rope_attn_get_device_status()
        ra.rope_attn_decode(q[:, :, :1].contiguous(), k, v, 500000.0, 1023)
        st2 = ra.rope_attn_get_device_status()
    finally:
        ra.rope_attn_set_wait_limit(old)
    assert st1 == ra.RA_ERR_DEVICE_TIMEOUT
    assert st2 == ra.RA_ERR_DEVICE_TIMEOUT
    again = ra.rope_attn_fwd(q, k, v, 500000.0)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    assert torch.equal(again, good)


def test_profile_pause_records_nothing():
    # a paused session records no kernel events, keeps what it had and resumes counting;
    # the paused call's output equals the profiled one
    q, k, v = rnd(1, 4, 300, 128, seed=40), rnd(1, 2, 300, 128, seed=41), rnd(1, 2, 300, 128, seed=42)
    qd, kd, vd = rnd(2, 8, 1, 128, seed=43), rnd(2, 2, 512, 128, seed=44), rnd(2, 2, 512, 128, seed=45)
    ra.rope_attn_profile_enable(True)
    try:
        o1 = ra.rope_attn_fwd(q, k, v, 10000.0)
        d1 = ra.rope_attn_decode(qd, kd, vd, 10000.0, 511)
        ra.rope_attn_profile_pause(True)
        o2 = ra.rope_attn_fwd(q, k, v, 10000.0)
        d2 = ra.rope_attn_decode(qd, kd, vd, 10000.0, 511)
        ra.rope_attn_profile_pause(False)
        o3 = ra.rope_attn_fwd(q, k, v, 10000.0)
        torch.cuda.synchronize()
        ms0, n0 = ra.rope_attn_profile_read(0)
        ms1, n1 = ra.rope_attn_profile_read(1)
    finally:
        ra.rope_attn_profile_enable(False)
    assert (n0, n1) == (2, 1)
    assert ms0 > 0 and ms1 > 0
    assert torch.equal(o1, o2) and torch.equal(o1, o3) and torch.equal(d1, d2)
