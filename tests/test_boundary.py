"""The C-ABI boundary, host side only (no kernel is launched here).

* the library loads and exports every function include/ropeattn.h declares, and the
  ctypes binding declares exactly those;
* invalid arguments come back as the documented status before any CUDA call, so these
  run on a machine without a GPU (device pointers are fake and never dereferenced).
"""
import ctypes
import os
import re

import pytest

import transformer_attention_04_b200 as ra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ropeattn.h")

FAKE = 0x10000  # 16-byte aligned, never dereferenced on the host


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rope_attn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(ra.LIB_PATH):
        from transformer_attention_04_b200 import build
        build.build()
    return ra.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(ra.SIGNATURES) == names
    assert lib.rope_attn_version() == 100


def test_status_strings(lib):
    for s in range(5):
        assert lib.rope_attn_status_string(s)
    assert b"invalid" in lib.rope_attn_status_string(1)


def test_wait_limit_roundtrip(lib):
    old = lib.rope_attn_set_wait_limit(12345)
    assert lib.rope_attn_set_wait_limit(-1) == 12345
    lib.rope_attn_set_wait_limit(old)
    assert lib.rope_attn_set_wait_limit(-1) == old


def fwd(lib, q=FAKE, k=FAKE + (1 << 40), v=FAKE + (2 << 40), out=FAKE + (3 << 40), B=1, Hq=4,
        Hkv=2, Sq=16, Sk=16, D=64, base=10000.0, pos=0, causal=1):
    return lib.rope_attn_fwd(q, k, v, out, B, Hq, Hkv, Sq, Sk, D, base, pos, causal, None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=0), ra.RA_ERR_INVALID_ARG),
    (dict(out=0), ra.RA_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), ra.RA_ERR_INVALID_ARG),          # misaligned
    (dict(Hq=3, Hkv=2), ra.RA_ERR_INVALID_ARG),         # Hq % Hkv != 0
    (dict(Sq=17, Sk=16), ra.RA_ERR_INVALID_ARG),        # causal with Sq > Sk
    (dict(B=0), ra.RA_ERR_INVALID_ARG),
    (dict(Sk=0), ra.RA_ERR_INVALID_ARG),
    (dict(base=0.0), ra.RA_ERR_INVALID_ARG),
    (dict(base=float("inf")), ra.RA_ERR_INVALID_ARG),
    (dict(pos=-1), ra.RA_ERR_INVALID_ARG),
    (dict(pos=2**31 - 8), ra.RA_ERR_INVALID_ARG),       # positions overflow int32
    (dict(out=FAKE), ra.RA_ERR_INVALID_ARG),            # out aliases q
    (dict(D=96), ra.RA_ERR_UNSUPPORTED),
    (dict(D=32), ra.RA_ERR_UNSUPPORTED),
])
def test_fwd_rejects(lib, kw, want):
    assert fwd(lib, **kw) == want


def test_fwd_noncausal_allows_sq_gt_sk_until_device(lib):
    # Sq > Sk is valid without the mask; with no GPU the call then fails at the device step
    st = fwd(lib, Sq=17, Sk=16, causal=0)
    assert st in (ra.RA_ERR_CUDA, ra.RA_ERR_UNSUPPORTED, ra.RA_OK)
    assert st != ra.RA_ERR_INVALID_ARG


def dec(lib, q=FAKE, k=FAKE + (1 << 40), v=FAKE + (2 << 40), out=FAKE + (3 << 40), B=2, Hq=8,
        Hkv=2, Sk=64, D=128, base=1e4, pos=63, splits=0):
    return lib.rope_attn_decode(q, k, v, out, B, Hq, Hkv, Sk, D, base, pos, splits, None)


@pytest.mark.parametrize("kw,want", [
    (dict(q=0), ra.RA_ERR_INVALID_ARG),
    (dict(v=FAKE + 4), ra.RA_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), ra.RA_ERR_INVALID_ARG),
    (dict(pos=-1), ra.RA_ERR_INVALID_ARG),
    (dict(splits=-2), ra.RA_ERR_INVALID_ARG),
    (dict(Sk=0), ra.RA_ERR_INVALID_ARG),
    (dict(out=FAKE + (1 << 40)), ra.RA_ERR_INVALID_ARG),  # out aliases the key cache
    (dict(D=80), ra.RA_ERR_UNSUPPORTED),
    (dict(B=40000, Hkv=2, Hq=2), ra.RA_ERR_UNSUPPORTED),  # grid.y over 65535
])
def test_decode_rejects(lib, kw, want):
    assert dec(lib, **kw) == want


@pytest.mark.parametrize("args,want", [
    ((0, FAKE, 1, 1, 8, 64, 1e4, 0), ra.RA_ERR_INVALID_ARG),
    ((FAKE, FAKE, 1, 1, 8, 6, 1e4, 0), ra.RA_ERR_INVALID_ARG),      # D % 8
    ((FAKE, FAKE, 1, 1, 8, 64, -1.0, 0), ra.RA_ERR_INVALID_ARG),
    ((FAKE, FAKE + 16, 1, 1, 8, 64, 1e4, 0), ra.RA_ERR_INVALID_ARG),  # partial overlap
    ((FAKE, FAKE, 1, 1, 8, 64, 1e4, -3), ra.RA_ERR_INVALID_ARG),
])
def test_rotate_rejects(lib, args, want):
    assert lib.rope_attn_rotate(*args, None) == want


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from transformer_attention_04_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def test_auto_splits_without_gpu(lib):
    # falls back to a 148-SM count when no device answers; always within [1, keys/64]
    s = lib.rope_attn_decode_auto_splits(32, 64, 8, 8192, 128, 8191)
    assert 1 <= s <= 128
    assert lib.rope_attn_decode_auto_splits(1, 1, 1, 10, 128, 9) == 1
