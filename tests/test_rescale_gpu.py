"""GPU parity on inputs that drive the online-softmax rescale of the prefill kernel.

On iid N(0, 1) inputs a row's maximum never grows by more than the kernel's threshold
after the first key tile, so the rescale of the running output and sum (and the redo of a
tile whose speculative P overflowed) never runs. The inputs of spike_cases.py plant keys in
later tiles that raise some rows' maxima by about 10, 40 and 140 (log2 units), on some lanes
of each warp and not on others, in masked and unmasked tiles. test_rescale_model.py shows on
the CPU that these inputs reach the branch and that a mistake in it would miss the bar.

Covered: causal prefill at D = 128 and 64, unmasked prefill with Sq < Sk, a sliding window,
a ring-attention block merged into an accumulator (rope_attn_fwd_partial with accumulate),
and a chunked prefill into a KV cache. Every output element is compared with the fp64
oracle at the usual bar (max-abs <= 2e-2, rel-RMS <= 5e-3); the block's LSE at max-abs
<= 2e-2.

Passage: "Transformer Architecture & Self-Attention Mechanics" §4 "The Quadratic
Bottleneck & FlashAttention" (running maximum, incremental rescaling).
"""
import numpy as np
import pytest
import torch

import transformer_attention_04_b200 as ra
from parity_util import assert_parity
from spike_cases import BASE, CASES, case_inputs, oracle_expected, rotated_keys_bf16

pytestmark = pytest.mark.gpu

LSE_MAX_ABS = 2e-2


def _ok():
    torch.cuda.synchronize()
    st = ra.rope_attn_get_device_status()
    assert st == ra.RA_OK, ra.lib().rope_attn_last_cuda_error()


@pytest.mark.parametrize("c", CASES, ids=[c.name for c in CASES])
def test_rescale_parity(c):
    q, k, v = case_inputs(c)
    want, want_lse = oracle_expected(c, q, k, v)
    gq, gk, gv = q.cuda(), k.cuda(), v.cuda()
    if c.kind == "prefill":
        out = ra.rope_attn_prefill(gq, gk, gv, BASE, 0, c.causal, window=c.window)
        _ok()
        assert_parity(out, want, c.name)
    elif c.kind == "partial":
        kr = rotated_keys_bf16(k).cuda()
        o_acc = torch.zeros(c.B, c.Hq, c.Sq, c.D, dtype=torch.float32, device="cuda")
        lse = torch.zeros(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
        out = torch.full((c.B, c.Hq, c.Sq, c.D), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        # the past block, then the diagonal block merged into it (views of the key tensors)
        ra.rope_attn_fwd_partial(gq, kr[:, :, :c.Sk], gv[:, :, :c.Sk], o_acc, lse, BASE,
                                 c.q_pos0, 0, c.causal, accumulate=False)
        ra.rope_attn_fwd_partial(gq, kr[:, :, c.Sk:], gv[:, :, c.Sk:], o_acc, lse, BASE,
                                 c.q_pos0, c.Sk, c.causal, accumulate=True, out=out)
        _ok()
        assert_parity(o_acc, want, c.name + " o_acc")
        assert_parity(out, want, c.name + " out")
        err = float(np.max(np.abs(lse.double().cpu().numpy() - want_lse)))
        assert err <= LSE_MAX_ABS, f"lse max_abs={err:.3e}"
    else:
        cap = c.P + c.Sk + 64
        kc = torch.full((c.B, c.Hkv, cap, c.D), float("nan"), dtype=torch.bfloat16)
        vc = kc.clone()
        kc[:, :, :c.P] = rotated_keys_bf16(k[:, :, :c.P])
        vc[:, :, :c.P] = v[:, :, :c.P]
        kc, vc = kc.cuda(), vc.cuda()
        out = ra.rope_attn_prefill(gq, gk[:, :, c.P:].contiguous(), gv[:, :, c.P:].contiguous(),
                                   BASE, c.P, c.causal, window=c.window, k_cache_rot=kc,
                                   v_cache=vc)
        _ok()
        assert_parity(out, want, c.name)


def test_rescale_rows_differ_from_unspiked():
    # the planted keys change the rows that see them by far more than the bar: a kernel that
    # ignored the jump would not pass the parity test above
    c = CASES[0]
    q, k, v = case_inputs(c)
    out = ra.rope_attn_prefill(q.cuda(), k.cuda(), v.cuda(), BASE, 0, True)
    k0 = k.clone()
    k0[..., -2:] = 0
    out0 = ra.rope_attn_prefill(q.cuda(), k0.cuda(), v.cuda(), BASE, 0, True)
    _ok()
    rows = torch.arange(c.Sq, device="cuda")
    sel = (rows % 4 == 0) & (rows >= 273)
    d = (out - out0).float()[:, :, sel].abs().amax()
    assert d > 0.5
