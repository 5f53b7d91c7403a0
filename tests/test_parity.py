"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same
seeded inputs. Bar: max-abs <= 2e-2 and relative RMS <= 5e-3 (bf16 in, fp32 accumulate).

Small problems are compared element by element over the whole output; the two large
prefill workloads are run in full on the GPU in the launch configuration the bench times
and compared on sampled query rows (all heads), which the oracle computes exactly since
every row of attention is independent.
"""
import numpy as np
import pytest
import torch

import oracle
import transformer_attention_04_b200 as ra
from synthetic import CONFIGS, Workload, make_inputs, to_f64
from parity_util import assert_parity, sample_rows

pytestmark = pytest.mark.gpu


def _run_fwd(w: Workload, seed=0):
    q, k, v = make_inputs(w, seed)
    out = ra.rope_attn_fwd(q.cuda(), k.cuda(), v.cuda(), w.rope_base, w.pos_offset, w.causal)
    torch.cuda.synchronize()
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    return q, k, v, out


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_config_full(name):
    w = CONFIGS[name]
    q, k, v, out = _run_fwd(w)
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), w.rope_base, w.pos_offset, w.causal)
    assert_parity(out, want, name)


@pytest.mark.parametrize("name", ["llama", "long"])
def test_config_sampled_rows(name):
    w = CONFIGS[name]
    q, k, v, out = _run_fwd(w)
    rows = sample_rows(w.Sq, block=64 if name == "llama" else 32, n_mid=3 if name == "llama" else 2)
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), w.rope_base, w.pos_offset,
                                w.causal, rows=rows)
    assert_parity(out[:, :, torch.from_numpy(rows).cuda()], want, name)


def test_config_decode():
    w = CONFIGS["decode"]
    q, kc, vc = make_inputs(w, 0)
    out = ra.rope_attn_decode(q.cuda(), kc.cuda(), vc.cuda(), w.rope_base, w.decode_pos)
    torch.cuda.synchronize()
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    want = oracle.rope_attn_decode(to_f64(q), to_f64(kc), to_f64(vc), w.rope_base, w.decode_pos)
    assert_parity(out, want, "decode")


# ragged and edge shapes: (B, Hq, Hkv, Sq, Sk, D, causal, pos_offset)
RAGGED = [
    (1, 1, 1, 1, 1, 64, True, 0),        # single row, single key
    (1, 2, 1, 1, 1, 128, True, 5),
    (1, 2, 2, 127, 127, 64, True, 0),    # one partial tile
    (1, 2, 2, 129, 129, 128, True, 0),   # one full tile plus one row
    (2, 4, 2, 1000, 1000, 128, True, 0),  # several tiles and a ragged tail, GQA G=2
    (1, 8, 1, 300, 300, 64, True, 0),    # MQA (one KV head), G=8
    (1, 3, 1, 200, 200, 128, True, 0),   # odd group size: one query tile per CTA
    (1, 6, 2, 257, 257, 64, True, 0),    # odd group size 3
    (1, 4, 2, 100, 700, 128, True, 11),  # Sq < Sk (bottom-right), pos_offset
    (1, 4, 4, 1, 513, 64, True, 0),      # one query row against many keys
    (2, 4, 2, 333, 333, 128, False, 0),  # no mask
    (1, 2, 1, 200, 77, 64, False, 3),    # no mask, Sq > Sk
    (1, 4, 1, 640, 640, 128, True, 0),   # exact multiple of the tile
    # long key ranges: 64 KV tiles per unit, so the K/V ring's slots are reused many times
    # (D = 64 keeps K and V in separate slots of an 8-slot ring, D = 128 alternates them in 3)
    (1, 4, 2, 256, 8192, 64, False, 0),
    (1, 4, 2, 256, 8192, 128, False, 0),
    (1, 3, 1, 256, 8192, 64, False, 0),  # odd group size: two query tiles per unit
    (1, 4, 2, 2048, 2048, 64, True, 0),
]


@pytest.mark.parametrize("shape", RAGGED, ids=[str(s) for s in RAGGED])
def test_ragged(shape):
    B, Hq, Hkv, Sq, Sk, D, causal, off = shape
    w = Workload("ragged", B, Hq, Hkv, Sq, Sk, D, 10000.0 if D == 64 else 500000.0, causal, off)
    q, k, v, out = _run_fwd(w, seed=7)
    want = oracle.rope_attn_fwd(to_f64(q), to_f64(k), to_f64(v), w.rope_base, off, causal)
    assert_parity(out, want, str(shape))


# decode shapes: (B, Hq, Hkv, Sk, D, pos, n_splits)
DECODE = [
    (1, 1, 1, 1, 64, 0, 0),
    (2, 8, 2, 100, 128, 99, 0),      # L = 100: ragged last tile
    (2, 8, 2, 100, 128, 40, 0),      # pos < Sk - 1: rows past pos ignored
    (1, 16, 1, 1000, 128, 999, 3),   # G = 16: two head blocks
    (3, 6, 2, 700, 64, 699, 5),      # G = 3: padded head block
    (1, 8, 8, 4096, 128, 4095, 1),   # single split
    (1, 64, 8, 2048, 128, 2047, 0),
]


@pytest.mark.parametrize("shape", DECODE, ids=[str(s) for s in DECODE])
def test_decode_shapes(shape):
    B, Hq, Hkv, Sk, D, pos, ns = shape
    w = Workload("dec", B, Hq, Hkv, 1, Sk, D, 500000.0, decode_pos=pos)
    q, kc, vc = make_inputs(w, 3)
    out = ra.rope_attn_decode(q.cuda(), kc.cuda(), vc.cuda(), w.rope_base, pos, n_splits=ns)
    torch.cuda.synchronize()
    assert ra.rope_attn_get_device_status() == ra.RA_OK
    want = oracle.rope_attn_decode(to_f64(q), to_f64(kc), to_f64(vc), w.rope_base, pos)
    assert_parity(out, want, str(shape))


def test_rotate_matches_oracle():
    gen = torch.Generator().manual_seed(5)
    x = torch.randn(2, 3, 1000, 128, generator=gen).to(torch.bfloat16)
    for base, off in ((10000.0, 0), (500000.0, 31000)):
        y = ra.rope_attn_rotate(x.cuda(), base, off)
        want = oracle.rope_rotate(to_f64(x), off + np.arange(1000), base)
        # one bf16 rounding of values of size ~|x|: half an ulp at 4 is 1.6e-2
        d = np.abs(y.double().cpu().numpy() - want)
        assert d.max() <= 1.6e-2 and np.sqrt((d ** 2).mean()) <= 3e-3
