"""Canaries in place of a memory checker (which this GPU pool does not offer): every output
sits inside a larger buffer whose guard regions hold a bit pattern that must survive the
call; every output starts as NaN, so an element the kernels fail to write shows; every input
must come back bit-identical. Ragged shapes, so tile tails and edge pages are exercised.
"""
import pytest
import torch

import transformer_attention_04_b200 as ra

pytestmark = pytest.mark.gpu

GUARD = 4096  # bf16 elements (8 KiB) on each side; a multiple of 8 keeps 16-byte alignment


def _bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16).cuda()


class Guarded:
    """A contiguous bf16 tensor of `shape` inside a buffer with guard regions around it,
    pre-filled with NaN (the guards with a fixed bit pattern)."""

    def __init__(self, shape):
        n = 1
        for d in shape:
            n *= d
        self.n = n
        self.buf = torch.empty(n + 2 * GUARD, dtype=torch.bfloat16, device="cuda")
        self.buf.view(torch.int16).fill_(0x5A5A)
        self.t = self.buf[GUARD:GUARD + n].view(*shape)
        self.t.fill_(float("nan"))

    def check(self, what):
        torch.cuda.synchronize()
        g = self.buf.view(torch.int16)
        assert bool((g[:GUARD] == 0x5A5A).all()), f"{what}: write before the output"
        assert bool((g[GUARD + self.n:] == 0x5A5A).all()), f"{what}: write past the output"
        assert not bool(torch.isnan(self.t.float()).any()), f"{what}: output element not written"


def _same(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("shape", [(2, 6, 2, 333, 700, 128, 7, 0), (1, 4, 4, 129, 129, 64, 0, 0),
                                   (1, 8, 2, 1, 513, 128, 3, 0), (2, 4, 2, 300, 300, 128, 0, 37)])
def test_prefill_guards(shape):
    B, Hq, Hkv, Sq, Sk, D, off, W = shape
    q, k, v = _bf16((B, Hq, Sq, D), 1), _bf16((B, Hkv, Sk, D), 2), _bf16((B, Hkv, Sk, D), 3)
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    o = Guarded((B, Hq, Sq, D))
    ra.rope_attn_prefill(q, k, v, 10000.0, off, True, window=W, out=o.t)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    o.check("prefill")
    assert _same(q, q0) and _same(k, k0) and _same(v, v0)


def test_prefill_into_cache_guards():
    B, Hq, Hkv, Sq, Sk, D, P, cap = 2, 4, 2, 200, 200, 128, 77, 300
    q, k, v = _bf16((B, Hq, Sq, D), 4), _bf16((B, Hkv, Sk, D), 5), _bf16((B, Hkv, Sk, D), 6)
    kc, vc = Guarded((B, Hkv, cap, D)), Guarded((B, Hkv, cap, D))
    kc.t.zero_()
    vc.t.zero_()
    o = Guarded((B, Hq, Sq, D))
    ra.rope_attn_prefill(q, k, v, 10000.0, P, True, k_cache_rot=kc.t, v_cache=vc.t, out=o.t)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    o.check("prefill into cache")
    kc.check("key cache")
    vc.check("value cache")


def test_rotate_guards():
    x = _bf16((2, 3, 129, 128), 7)
    x0 = x.clone()
    o = Guarded((2, 3, 129, 128))
    ra.rope_attn_rotate(x, 10000.0, 5, out=o.t)
    o.check("rotate")
    assert _same(x, x0)


@pytest.mark.parametrize("n_splits", [0, 1, 7])
def test_decode_guards(n_splits):
    B, Hq, Hkv, Sk, D = 3, 12, 3, 1000, 128
    q, kc, vc = _bf16((B, Hq, 1, D), 8), _bf16((B, Hkv, Sk, D), 9), _bf16((B, Hkv, Sk, D), 10)
    kc0, vc0 = kc.clone(), vc.clone()
    o = Guarded((B, Hq, 1, D))
    ra.rope_attn_decode(q, kc, vc, 10000.0, 900, n_splits=n_splits, out=o.t)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    o.check("decode")
    assert _same(kc, kc0) and _same(vc, vc0)


def test_decode_step_and_paged_guards():
    B, Hq, Hkv, cap, D, page = 3, 8, 2, 256, 64, 16
    q = _bf16((B, Hq, 1, D), 11)
    kn, vn = _bf16((B, Hkv, 1, D), 12), _bf16((B, Hkv, 1, D), 13)
    pos = torch.tensor([255, 0, 100], dtype=torch.int32, device="cuda")
    kc, vc = Guarded((B, Hkv, cap, D)), Guarded((B, Hkv, cap, D))
    kc.t.copy_(_bf16((B, Hkv, cap, D), 14))
    vc.t.copy_(_bf16((B, Hkv, cap, D), 15))
    o = Guarded((B, Hq, 1, D))
    ra.rope_attn_decode_step(q, kc.t, vc.t, pos, 255, 10000.0, kn, vn, window=30, out=o.t)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    o.check("decode step")
    kc.check("key cache")
    vc.check("value cache")

    nb = B * cap // page
    pk, pv = Guarded((nb, Hkv, page, D)), Guarded((nb, Hkv, page, D))
    pk.t.copy_(_bf16((nb, Hkv, page, D), 16))
    pv.t.copy_(_bf16((nb, Hkv, page, D), 17))
    table = torch.randperm(nb, generator=torch.Generator().manual_seed(18)).view(B, -1)
    table = table.to(torch.int32).cuda()
    t0 = table.clone()
    o2 = Guarded((B, Hq, 1, D))
    ra.rope_attn_decode_paged(q, pk.t, pv.t, table, pos, 255, 10000.0, kn, vn, out=o2.t)
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    o2.check("paged decode")
    pk.check("key pool")
    pv.check("value pool")
    assert torch.equal(table, t0)
