"""The spike inputs reach the online-softmax rescale, and a mistake there would fail parity.

The GPU tests of test_rescale_gpu.py compare the kernel with the oracle on the inputs of
spike_cases.py. This CPU test runs a model of the kernel's tile loop (rescale_model.py) on
the same inputs and shows, for every case:

* the rescale fires on many rows after their first tile, on lanes of the same warp that
  disagree, in masked and unmasked tiles, and (for the largest jump) with a speculative
  P = 2^(s - m_old) that overflows fp32 and must be redone;
* the model without a mistake meets the parity bar against the oracle;
* the model with one planted mistake (l not rescaled, O not rescaled, or the tile not
  redone after a jump) misses the bar by a wide margin, so the GPU test on the same inputs
  and bar would catch that mistake in the kernel.

The online softmax is "Transformer Architecture & Self-Attention Mechanics" §4 "The
Quadratic Bottleneck & FlashAttention" (running maximum, incremental rescaling).
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import MAX_ABS, REL_RMS, errors
from rescale_model import merge, model_call
from spike_cases import BASE, CASES, case_inputs, oracle_expected, rotated_keys_bf16

BUGS = ("l_alpha", "o_alpha", "no_redo")


def _model(c, q, k, v, bugs=()):
    """Run the model over every (batch, head) of the case; returns (out, stats)."""
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    q64, v64 = f(q), f(v)
    G = c.Hq // c.Hkv
    out = np.zeros(q64.shape)
    tot = {}
    if c.kind == "prefill":
        k_rot = oracle.rope_rotate(f(k), np.arange(c.Sk), BASE)
        q_rot = oracle.rope_rotate(q64, oracle.query_positions(c.Sq, c.Sk, 0), BASE)
    elif c.kind == "partial":
        k_rot = f(rotated_keys_bf16(k))
        q_rot = oracle.rope_rotate(q64, c.q_pos0 + np.arange(c.Sq), BASE)
    else:
        n = c.P + c.Sk
        k_rot = oracle.rope_rotate(f(k), np.arange(n), BASE)
        q_rot = oracle.rope_rotate(q64, oracle.query_positions(c.Sq, n, 0), BASE)
    for b in range(c.B):
        for h in range(c.Hq):
            kv = h // G
            if c.kind == "prefill":
                o, _, st = model_call(q_rot[b, h], k_rot[b, kv], v64[b, kv], c.causal,
                                      c.Sk - c.Sq, c.window, bugs)
            elif c.kind == "partial":
                o1, l1, st = model_call(q_rot[b, h], k_rot[b, kv, :c.Sk], v64[b, kv, :c.Sk],
                                        c.causal, c.q_pos0, 0, bugs)
                o2, l2, st2 = model_call(q_rot[b, h], k_rot[b, kv, c.Sk:], v64[b, kv, c.Sk:],
                                         c.causal, c.q_pos0 - c.Sk, 0, bugs)
                o, _ = merge(o1, l1, o2, l2)
                st = {key: st[key] + st2[key] for key in st}
            else:
                o, _, st = model_call(q_rot[b, h], k_rot[b, kv], v64[b, kv], c.causal,
                                      c.P + c.Sk - c.Sq, c.window, bugs)
            out[b, h] = o
            for key, val in st.items():
                tot[key] = tot.get(key, 0) + val
    return out, tot


@pytest.mark.parametrize("c", CASES, ids=[c.name for c in CASES])
def test_spike_inputs_reach_the_rescale(c):
    q, k, v = case_inputs(c)
    want, _ = oracle_expected(c, q, k, v)
    got, st = _model(c, q, k, v)
    rows = c.B * c.Hq * c.Sq
    # the branch fires on a good share of rows, in masked and unmasked tiles, and the largest
    # jump overflows the speculative P
    assert st["rows_rescaled"] >= rows // 16, st
    assert st["rescale"] > st["rescale_masked"] > 0, st
    assert st["overflow"] > 0, st
    # lanes of one warp disagree: rows with a = 8 rescale, rows with a = 0 (iid scores) never
    by_lane = st["row_mod4_rescaled"]
    assert by_lane[0] > 0 and by_lane[3] == 0, by_lane
    ma, rr = errors(got, want)
    assert ma <= MAX_ABS and rr <= REL_RMS, (ma, rr)
    for bug in BUGS:
        bad, _ = _model(c, q, k, v, bugs=(bug,))
        with np.errstate(invalid="ignore"):
            ma, rr = errors(bad, want)
        assert not (ma <= 4 * MAX_ABS and rr <= 4 * REL_RMS), (bug, ma, rr)


def test_iid_inputs_never_rescale_after_the_first_tile():
    # the reason the spike inputs exist: on N(0,1) data the branch stays cold
    g = torch.Generator().manual_seed(0)
    q = torch.randn(1, 1, 1024, 128, generator=g).double().numpy()
    k = torch.randn(1, 1, 1024, 128, generator=g).double().numpy()
    v = torch.randn(1, 1, 1024, 128, generator=g).double().numpy()
    pos = np.arange(1024)
    _, _, st = model_call(oracle.rope_rotate(q, pos, BASE)[0, 0],
                          oracle.rope_rotate(k, pos, BASE)[0, 0], v[0, 0], True, 0)
    assert st["rescale"] == 0
