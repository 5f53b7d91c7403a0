"""rope_attn_decode_noalloc: the decode step for callers that may not allocate device memory
while they run it (for instance a serving process that has reserved the GPU's memory for its
own pool and does not let libraries take more, or a step that must not stall or fail on an
allocation). The entry keeps its per-split partials in one fixed 16 MiB device array of the
library instead of memory taken per call.

The test calls the entry through the C ABI twice in a row, on different inputs (so a stale
partial left by the first call would show in the second), and compares each result with the
allocating rope_attn_decode within the parity tolerance of the other tests, and once directly
with the fp64 oracle. It also checks that the automatic split count's partials fit the
array for large head counts (the contiguous-cache policy takes the fewest splits that put two
CTAs on every SM, so many heads mean one split), that the result then equals the allocating
decode with that count, and that a request whose partials cannot fit the array, even with
one split, is refused before anything is enqueued.
The file is named to be collected last.
"""
import ctypes

import pytest
import torch

import oracle
import transformer_attention_04_b200 as ra
from parity_util import MAX_ABS, REL_RMS, assert_parity, errors

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _inputs(seed, B, Hq, Hkv, Sk, D):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, 1, D, generator=g).to(torch.bfloat16).cuda()
    kc = torch.randn(B, Hkv, Sk, D, generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn(B, Hkv, Sk, D, generator=g).to(torch.bfloat16).cuda()
    return q, kc, vc


def _noalloc(q, kc, vc, base, pos, n_splits):
    B, Hq, _, D = q.shape
    Hkv, Sk = kc.shape[1], kc.shape[2]
    out = torch.empty_like(q)
    st = ra.lib().rope_attn_decode_noalloc(
        q.data_ptr(), kc.data_ptr(), vc.data_ptr(), out.data_ptr(), B, Hq, Hkv, Sk, D, base, pos,
        n_splits, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


@pytest.mark.parametrize("shape", [(4, 16, 2, 3000, 128, 2999, 0), (2, 8, 8, 777, 64, 700, 3),
                                   (32, 64, 8, 8192, 128, 8191, 0)])
def test_noalloc_matches_decode_twice(shape):
    B, Hq, Hkv, Sk, D, pos, ns = shape
    base = 500000.0
    for call, seed in enumerate((11, 12)):
        q, kc, vc = _inputs(seed, B, Hq, Hkv, Sk, D)
        ref = ra.rope_attn_decode(q, kc, vc, base, pos, n_splits=ns)
        st, out = _noalloc(q, kc, vc, base, pos, ns)
        assert st == ra.RA_OK, ra.lib().rope_attn_last_cuda_error()
        torch.cuda.synchronize()
        assert ra.rope_attn_get_device_status() == ra.RA_OK
        ma, rr = errors(out, ref.double().cpu().numpy())
        assert ma <= MAX_ABS and rr <= REL_RMS, (call, ma, rr)


def _partials_bytes(B, Hq, D, splits):
    rows = B * Hq * splits
    return ((rows * D * 4 + 255) & ~255) + rows * 8


def test_noalloc_matches_oracle():
    B, Hq, Hkv, Sk, D, pos = 4, 16, 2, 3000, 128, 2999
    q, kc, vc = _inputs(13, B, Hq, Hkv, Sk, D)
    st, out = _noalloc(q, kc, vc, 500000.0, pos, 0)
    assert st == ra.RA_OK, ra.lib().rope_attn_last_cuda_error()
    torch.cuda.synchronize()
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    f = lambda t: t.double().cpu().numpy()  # noqa: E731
    assert_parity(out, oracle.rope_attn_decode(f(q), f(kc), f(vc), 500000.0, pos), "noalloc")


def test_noalloc_automatic_split_count_fits():
    # 21 x 800 query heads: 2100 (batch, KV head, 8-head block) CTAs already fill a 148-SM
    # B200, so the automatic count is 1 and its partials (8.3 MiB) fit; the entry must then
    # give what the allocating decode gives with that count. Over the shapes below, the
    # automatic count's partials never exceed the array
    B, Hq, Hkv, Sk, D, pos = 21, 800, 10, 128, 128, 127
    auto = ra.rope_attn_decode_auto_splits(B, Hq, Hkv, Sk, D, pos)
    assert _partials_bytes(B, Hq, D, auto) <= SCRATCH_BYTES
    for shape in ((32, 64, 8, 8192), (1, 8, 8, 131072), (1, 64, 1, 65536), (4, 128, 128, 4096),
                  (64, 32, 32, 2048)):
        b, hq, hkv, sk = shape
        a = ra.rope_attn_decode_auto_splits(b, hq, hkv, sk, D, sk - 1)
        assert _partials_bytes(b, hq, D, a) <= SCRATCH_BYTES, (shape, a)
    for seed in (14, 15):
        q, kc, vc = _inputs(seed, B, Hq, Hkv, Sk, D)
        ref = ra.rope_attn_decode(q, kc, vc, 500000.0, pos, n_splits=auto)
        st, out = _noalloc(q, kc, vc, 500000.0, pos, 0)
        assert st == ra.RA_OK, ra.lib().rope_attn_last_cuda_error()
        torch.cuda.synchronize()
        assert ra.rope_attn_get_device_status() == ra.RA_OK
        ma, rr = errors(out, ref.double().cpu().numpy())
        assert ma <= MAX_ABS and rr <= REL_RMS, (seed, ma, rr)


def test_noalloc_refuses_when_one_split_does_not_fit():
    # 128 x 256 heads need 16.25 MiB of partials even with a single split
    B, Hq, Hkv, Sk, D = 128, 256, 8, 64, 128
    assert _partials_bytes(B, Hq, D, 1) > SCRATCH_BYTES
    q = torch.zeros(B, Hq, 1, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(B, Hkv, Sk, D, dtype=torch.bfloat16, device="cuda")
    st, _ = _noalloc(q, kc, kc.clone(), 500000.0, Sk - 1, 0)
    assert st == ra.RA_ERR_UNSUPPORTED
    assert b"scratch" in ra.lib().rope_attn_last_cuda_error()


def test_noalloc_rejects_partials_beyond_scratch():
    # 64 x 256 heads x 8 splits x (128 x 4 + 8) bytes is about 68 MB, over the 16 MiB array
    B, Hq, Hkv, Sk, D, splits = 64, 256, 8, 1024, 128, 8
    q = torch.zeros(B, Hq, 1, D, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(B, Hkv, Sk, D, dtype=torch.bfloat16, device="cuda")
    st, _ = _noalloc(q, kc, kc.clone(), 500000.0, Sk - 1, splits)
    assert st == ra.RA_ERR_UNSUPPORTED
    assert b"scratch" in ra.lib().rope_attn_last_cuda_error()
    assert B * Hq * splits * (D * 4 + 8) > SCRATCH_BYTES
