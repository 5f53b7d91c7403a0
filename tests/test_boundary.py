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
    ((FAKE, FAKE, 1 << 16, 1 << 15, 1, 8, 1e4, 0), ra.RA_ERR_UNSUPPORTED),  # 2^31 heads
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
    # the contiguous cache takes the fewest splits that put two CTAs on each of 148 SMs:
    # 256 (batch, KV head) blocks need 2; 8 blocks need 37, capped at 32
    assert s == 2
    assert lib.rope_attn_decode_auto_splits(1, 8, 8, 8192, 128, 8191) == 32
    assert lib.rope_attn_decode_auto_splits(1, 8, 8, 1000, 128, 999) == 16  # keys / 64


def test_header_is_plain_c_and_links(tmp_path, lib):
    # include/ropeattn.h compiles as C99 with warnings as errors, and a C caller links
    # against the library (no C++ or CUDA types cross the boundary)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(
        '#include "ropeattn.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        "  ra_status s = rope_attn_fwd(0, 0, 0, 0, 1, 1, 1, 1, 1, 64, 10000.f, 0, 1, 0);\n"
        "  printf(\"%d %d %s\\n\", (int)s, rope_attn_version(), rope_attn_status_string(s));\n"
        "  return s == RA_ERR_INVALID_ARG ? 0 : 1;\n"
        "}\n")
    exe = tmp_path / "caller"
    libdir = os.path.dirname(ra.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir,
                        "-lropeattn", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert run.stdout.split()[1] == "100"


def prefill(lib, q=FAKE, k=FAKE + (1 << 40), v=FAKE + (2 << 40), out=FAKE + (3 << 40),
            kc=0, vc=0, S_cache=0, B=1, Hq=4, Hkv=2, Sq=16, Sk=16, D=64, base=10000.0, pos=0,
            causal=1, window=0):
    return lib.rope_attn_prefill(q, k, v, out, kc, vc, S_cache, B, Hq, Hkv, Sq, Sk, D, base, pos,
                                 causal, window, None)


@pytest.mark.parametrize("kw", [
    dict(window=-1),                                           # negative window
    dict(window=8, causal=0),                                  # a window needs the causal mask
    dict(kc=FAKE + (4 << 40)),                                 # one cache without the other
    dict(kc=FAKE + (4 << 40), vc=FAKE + (5 << 40), S_cache=0),  # caches without a row count
    dict(kc=FAKE + (4 << 40), vc=FAKE + (5 << 40), S_cache=20, pos=8),  # pos_offset + Sk > S_cache
    dict(kc=FAKE + (4 << 40) + 8, vc=FAKE + (5 << 40), S_cache=64),     # misaligned cache
    dict(kc=FAKE + (3 << 40), vc=FAKE + (5 << 40), S_cache=64),         # cache overlaps out
])
def test_prefill_rejects(lib, kw):
    assert prefill(lib, **kw) == ra.RA_ERR_INVALID_ARG


def step(lib, q=FAKE, kn=0, vn=0, kc=FAKE + (1 << 40), vc=FAKE + (2 << 40), out=FAKE + (3 << 40),
         pos=FAKE + (4 << 40), B=2, Hq=4, Hkv=2, S_cache=128, D=64, base=10000.0, max_pos=100,
         window=0, splits=0):
    return lib.rope_attn_decode_step(q, kn, vn, kc, vc, out, pos, B, Hq, Hkv, S_cache, D, base,
                                     max_pos, window, splits, None)


@pytest.mark.parametrize("kw", [
    dict(pos=0),                           # positions are required
    dict(max_pos=128),                     # positions must lie inside the cache
    dict(max_pos=-1),
    dict(kn=FAKE + (5 << 40)),             # new key without new value
    dict(window=-2),
    dict(splits=-1),
    dict(Hq=3),                            # Hq % Hkv != 0
])
def test_decode_step_rejects(lib, kw):
    assert step(lib, **kw) == ra.RA_ERR_INVALID_ARG


def paged(lib, q=FAKE, kp=FAKE + (1 << 40), vp=FAKE + (2 << 40), table=FAKE + (3 << 40),
          out=FAKE + (4 << 40), pos=FAKE + (5 << 40), B=2, Hq=4, Hkv=2, D=64, page=16, maxb=8,
          nb=16, base=10000.0, max_pos=100, window=0, splits=0):
    return lib.rope_attn_decode_paged(q, 0, 0, kp, vp, table, out, pos, B, Hq, Hkv, D, page, maxb,
                                      nb, base, max_pos, window, splits, None)


@pytest.mark.parametrize("kw", [
    dict(page=12),                         # pages must divide 64 ...
    dict(page=4),                          # ... and hold at least 8 rows
    dict(table=0),
    dict(max_pos=128),                     # 8 blocks x 16 rows hold positions 0..127
    dict(nb=0),
    dict(maxb=0),
])
def test_decode_paged_rejects(lib, kw):
    assert paged(lib, **kw) == ra.RA_ERR_INVALID_ARG


def partial(lib, q=FAKE, k=FAKE + (1 << 40), v=FAKE + (2 << 40), o=FAKE + (3 << 40),
            lse=FAKE + (4 << 40), out=0, B=1, Hq=4, Hkv=2, Sq=16, Sk=16, D=64, base=10000.0,
            qp=32, kp=16, causal=1, acc=0, q_rows=0, kv_rows=0, acc_rows=0, split=0, qp1=0):
    return lib.rope_attn_fwd_partial(q, k, v, o, lse, out, B, Hq, Hkv, Sq, Sk, D, base, qp, kp,
                                     causal, acc, q_rows, kv_rows, acc_rows, split, qp1, None)


@pytest.mark.parametrize("kw,want", [
    (dict(o=0), ra.RA_ERR_INVALID_ARG),                 # the accumulator is required
    (dict(lse=0), ra.RA_ERR_INVALID_ARG),
    (dict(o=FAKE + (3 << 40) + 4), ra.RA_ERR_INVALID_ARG),  # o_acc not 16-byte aligned
    (dict(lse=FAKE + (4 << 40) + 2), ra.RA_ERR_INVALID_ARG),  # lse_acc not 4-byte aligned
    (dict(qp=15, kp=16), ra.RA_ERR_INVALID_ARG),        # causal rows before the block's first key
    (dict(qp=-1), ra.RA_ERR_INVALID_ARG),
    (dict(qp=2**30, kp=0), ra.RA_ERR_INVALID_ARG),      # positions past 2^30
    (dict(Hq=3), ra.RA_ERR_INVALID_ARG),
    (dict(o=FAKE), ra.RA_ERR_INVALID_ARG),              # o_acc overlaps q
    (dict(lse=FAKE + (3 << 40)), ra.RA_ERR_INVALID_ARG),  # lse_acc overlaps o_acc
    (dict(out=FAKE + (2 << 40)), ra.RA_ERR_INVALID_ARG),  # out overlaps v
    (dict(D=96), ra.RA_ERR_UNSUPPORTED),
    (dict(q_rows=15), ra.RA_ERR_INVALID_ARG),           # head stride shorter than the rows
    (dict(kv_rows=-1), ra.RA_ERR_INVALID_ARG),
    (dict(acc_rows=8), ra.RA_ERR_INVALID_ARG),
    (dict(split=8, qp1=100), ra.RA_ERR_INVALID_ARG),    # masked: q_split not on a 128-row edge
    (dict(Sq=256, split=128, qp1=15, kp=16, qp=32), ra.RA_ERR_INVALID_ARG),  # 2nd segment early
    (dict(Sq=384, Hq=6, Hkv=2, split=128, qp1=500), ra.RA_ERR_INVALID_ARG),  # odd G: 256 rows
    (dict(split=8, qp1=-1, causal=0), ra.RA_ERR_INVALID_ARG),
    (dict(split=-1), ra.RA_ERR_INVALID_ARG),
    # o_acc inside k's strided extent (2 heads 64 rows apart: 80 rows of 128 bytes)
    (dict(kv_rows=64, o=FAKE + (1 << 40) + 8192), ra.RA_ERR_INVALID_ARG),
])
def test_partial_rejects(lib, kw, want):
    assert partial(lib, **kw) == want


def test_partial_noncausal_any_offsets_until_device(lib):
    # without the mask a block may sit anywhere; with no GPU the call fails at the device step
    st = partial(lib, qp=0, kp=500, causal=0)
    assert st != ra.RA_ERR_INVALID_ARG


def test_partial_masked_two_segments_until_device(lib):
    # a masked call with two query segments on 128-row edges passes the checks (odd G: 256)
    for kw in (dict(Sq=256, split=128, qp1=500), dict(Sq=512, Hq=6, Hkv=2, split=256, qp1=32)):
        assert partial(lib, **kw) != ra.RA_ERR_INVALID_ARG, kw


def test_view_rows_of_real_layouts():
    import torch
    # the binding's stride logic on CPU tensors of the layouts the entry points accept
    from transformer_attention_04_b200._lib import view_rows
    x = torch.empty(2, 3, 100, 64)
    assert view_rows(tuple(x.shape), x.stride()) == 100                      # packed
    v = x[:, :, 10:60]
    assert view_rows(tuple(v.shape), v.stride()) == 100                      # slice along S
    one = torch.empty(1, 5, 40, 64)[:, :, 8:24]
    assert view_rows(tuple(one.shape), one.stride()) == 40                   # B = 1
    single = torch.empty(3, 1, 40, 64)[:, :, :16]
    assert view_rows(tuple(single.shape), single.stride()) == 40             # H = 1
    lse = torch.empty(2, 3, 100)[:, :, 5:50]
    assert view_rows(tuple(lse.shape), lse.stride()) == 100                  # 3-D accumulator
    t = x.transpose(1, 2)                                                    # [B, S, H, D]
    assert view_rows((2, 100, 3, 64), t.stride()) is None
    cols = x[:, :, :, :32]                                                   # rows not packed
    assert view_rows(tuple(cols.shape), cols.stride()) is None
    heads = x[:, :2]                                                          # uneven batch step
    assert view_rows(tuple(heads.shape), heads.stride()) is None


def test_profile_pause_needs_a_session(lib):
    # disabling needs no device; a pause outside a session is refused
    assert lib.rope_attn_profile_enable(0) == ra.RA_OK
    assert lib.rope_attn_profile_pause(1) == ra.RA_ERR_INVALID_ARG
    assert lib.rope_attn_profile_pause(0) == ra.RA_ERR_INVALID_ARG
