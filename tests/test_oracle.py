"""Pins for the fp64 oracle: values the pages print, closed forms, invariants, an
independent brute force and a library cross-check. CPU only.

Each test targets a plausible mistake in the oracle (a wrong rotation sense, a
dropped 1/sqrt(D), a transposed operand, an off-by-one in the mask, a wrong head
map); ``test_planted_mistakes_are_caught`` plants such mistakes in a copy of the
oracle and checks that a pin fails for each.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
import oracle
from oracle import ref
from synthetic import TINY, Workload, make_inputs, to_f64


# ----------------------------------------------------------------- pages' values

def _weights_of_one_query(logits, d_k):
    """Attention weights of one query over len(logits) keys whose raw dot products
    with it are ``logits``: q = (c, 0, ...), key_j = (logit_j / c, 0, ...), V = identity."""
    n = len(logits)
    c = 4.0
    q = np.zeros((1, 1, 1, d_k))
    q[0, 0, 0, 0] = c
    k = np.zeros((1, 1, n, d_k))
    k[0, 0, :, 0] = np.asarray(logits) / c
    v = np.zeros((1, 1, n, n))
    v[0, 0] = np.eye(n)
    return oracle.attention(q, k, v, causal=False)[0, 0, 0]


def test_problem1_scaled_softmax_weights():
    g = read_golden("problem1_scaled_softmax.txt")
    w = _weights_of_one_query(g["logits"], int(g["d_k"]))
    np.testing.assert_allclose(w, g["scaled_weights"], atol=g["scaled_weights_tol"], rtol=0)


def test_problem1_unscaled_is_not_what_oracle_computes():
    # with d_k = 1 the 1/sqrt(d_k) factor is 1, which reproduces the page's unscaled row;
    # at d_k = 64 the oracle must NOT give it (pins that the scale is applied).
    g = read_golden("problem1_scaled_softmax.txt")
    w1 = _weights_of_one_query(g["logits"], 1)
    np.testing.assert_allclose(w1, g["unscaled_weights"], atol=g["unscaled_weights_tol"], rtol=0)
    w64 = _weights_of_one_query(g["logits"], 64)
    assert abs(w64[0] - g["unscaled_weights"][0]) > 0.3


def test_problem2_two_token_head():
    g = read_golden("problem2_head_output.txt")
    Q = np.array(g["Q1"])[None, None]
    K = np.array(g["K1"])[None, None]
    V = np.array(g["V1"])[None, None]
    H = oracle.attention(Q, K, V, causal=False)[0, 0]
    np.testing.assert_allclose(H, np.array(g["H1"]), atol=g["tol"], rtol=0)
    # the weights themselves: V = I returns A
    A = oracle.attention(Q, K, np.eye(2)[None, None], causal=False)[0, 0]
    np.testing.assert_allclose(A, np.array(g["A1"]), atol=g["tol"], rtol=0)


def test_problem3_rope_sign_pin():
    g = read_golden("problem3_rope_relative.txt")
    q = np.array(g["q"])[None, :]
    k = np.array(g["k"])[None, :]
    qr = oracle.rope_rotate(q, np.array([int(g["m"])]), 10000.0)
    kr = oracle.rope_rotate(k, np.array([int(g["n"])]), 10000.0)
    assert abs(float(qr[0] @ kr[0]) - g["value"]) < g["tol"]


@pytest.mark.parametrize("D,base", [(2, 10000.0), (8, 10000.0), (64, 10000.0), (128, 500000.0)])
def test_problem3_rope_closed_form_random(D, base):
    rng = np.random.default_rng(1)
    theta = base ** (-2.0 * np.arange(D // 2) / D)
    for _ in range(20):
        q, k = rng.standard_normal(D), rng.standard_normal(D)
        m, n = rng.integers(0, 40000, size=2)
        qr = oracle.rope_rotate(q[None], np.array([m]), base)[0]
        kr = oracle.rope_rotate(k[None], np.array([n]), base)[0]
        for i in range(D // 2):
            q1, q2, k1, k2 = q[2 * i], q[2 * i + 1], k[2 * i], k[2 * i + 1]
            dot, cross = q1 * k1 + q2 * k2, q2 * k1 - q1 * k2
            want = dot * math.cos((m - n) * theta[i]) - cross * math.sin((m - n) * theta[i])
            got = qr[2 * i] * kr[2 * i] + qr[2 * i + 1] * kr[2 * i + 1]
            assert abs(got - want) < 1e-9 * (1 + abs(dot) + abs(cross))


# ----------------------------------------------------------------- RoPE properties

def test_rope_position_zero_is_identity():
    # the page-5 demo rotates a token at position 0: R_0 = I
    x = np.random.default_rng(2).standard_normal((5, 64))
    np.testing.assert_array_equal(oracle.rope_rotate(x, np.zeros(5, dtype=np.int64), 10000.0), x)


@pytest.mark.parametrize("D,base", [(8, 10000.0), (64, 10000.0), (128, 500000.0)])
def test_rope_frequencies(D, base):
    # pair i of a unit vector along x_2i, at position 1, turns by exactly base^(-2i/D)
    x = np.zeros((D // 2, D))
    for i in range(D // 2):
        x[i, 2 * i] = 1.0
    r = oracle.rope_rotate(x, np.ones(D // 2, dtype=np.int64), base)
    for i in range(D // 2):
        ang = math.atan2(r[i, 2 * i + 1], r[i, 2 * i])
        assert abs(ang - base ** (-2.0 * i / D)) < 1e-14


def test_rope_is_complex_multiplication():
    # independent formulation: pair (x_2i, x_2i+1) as z = x_2i + i x_2i+1, times e^{i m theta}
    rng = np.random.default_rng(3)
    D, base = 64, 10000.0
    x = rng.standard_normal((7, D))
    pos = rng.integers(0, 100000, size=7)
    z = x[:, 0::2] + 1j * x[:, 1::2]
    theta = np.array([base ** (-2.0 * i / D) for i in range(D // 2)])
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    r = oracle.rope_rotate(x, pos, base)
    np.testing.assert_allclose(r[:, 0::2], zr.real, atol=1e-9)
    np.testing.assert_allclose(r[:, 1::2], zr.imag, atol=1e-9)
    # rotations keep norms
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


def test_relative_invariance_through_pos_offset():
    q, k, v = (to_f64(t) for t in make_inputs(Workload("t", 1, 2, 2, 48, 48, 16, 10000.0), seed=4))
    o0 = oracle.rope_attn_fwd(q, k, v, 10000.0, pos_offset=0)
    for c in (1, 17, 12345):
        oc = oracle.rope_attn_fwd(q, k, v, 10000.0, pos_offset=c)
        np.testing.assert_allclose(oc, o0, atol=1e-10, rtol=0)


# ----------------------------------------------------------------- attention invariants

def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_rows_sum_to_one():
    q, k = _rand((2, 4, 33, 16), 5), _rand((2, 2, 33, 16), 6)
    v = np.ones((2, 2, 33, 16))
    for causal in (True, False):
        o = oracle.rope_attn_fwd(q, k, v, 10000.0, causal=causal)
        np.testing.assert_allclose(o, 1.0, atol=1e-13)


def test_causal_row0_is_v0():
    q, k, v = _rand((1, 3, 40, 16), 7), _rand((1, 3, 40, 16), 8), _rand((1, 3, 40, 16), 9)
    o = oracle.rope_attn_fwd(q, k, v, 10000.0, causal=True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-14, rtol=0)


def test_zero_q_gives_prefix_mean():
    S = 50
    q = np.zeros((1, 2, S, 16))
    k, v = _rand((1, 2, S, 16), 10), _rand((1, 2, S, 16), 11)
    o = oracle.rope_attn_fwd(q, k, v, 10000.0, causal=True)
    prefix = np.cumsum(v, axis=2) / np.arange(1, S + 1)[None, None, :, None]
    np.testing.assert_allclose(o, prefix, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    q, k, v = _rand((2, 8, 30, 16), 12), _rand((2, 2, 30, 16), 13), _rand((2, 2, 30, 16), 14)
    o = oracle.rope_attn_fwd(q, k, v, 10000.0)
    o_mha = oracle.rope_attn_fwd(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), 10000.0)
    np.testing.assert_allclose(o, o_mha, atol=1e-13, rtol=0)
    # and the head map is contiguous: head 5 reads kv head 1, not kv head 5 % 2
    o_wrong = oracle.rope_attn_fwd(q, np.tile(k, (1, 4, 1, 1)), np.tile(v, (1, 4, 1, 1)), 10000.0)
    assert np.max(np.abs(o_wrong[:, 1] - o[:, 1])) > 1e-3


def test_permutation_equivariance():
    # without mask and rotation, attention(P X) = P attention(X): permuting keys and values
    # together leaves the output alone; permuting queries permutes the output
    q, k, v = _rand((1, 1, 12, 8), 15), _rand((1, 1, 12, 8), 16), _rand((1, 1, 12, 8), 17)
    p = np.random.default_rng(18).permutation(12)
    o = oracle.attention(q, k, v, causal=False)
    np.testing.assert_allclose(oracle.attention(q, k[:, :, p], v[:, :, p], causal=False), o, atol=1e-13)
    np.testing.assert_allclose(oracle.attention(q[:, :, p], k, v, causal=False), o[:, :, p], atol=1e-13)


def test_score_variance_is_one():
    # iid N(0,1) rotated q, k: q.k / sqrt(D) has mean 0 and variance 1 (devthesis §1)
    q, k, _ = (to_f64(t) for t in make_inputs(Workload("s", 1, 1, 1, 2048, 2048, 128, 500000.0), seed=19))
    pos = np.arange(2048)
    qr = oracle.rope_rotate(q[0, 0], pos, 500000.0)
    kr = oracle.rope_rotate(k[0, 0], pos, 500000.0)
    s = (qr @ kr.T).ravel() / math.sqrt(128)
    assert abs(s.mean()) < 0.01 and abs(s.var() - 1.0) < 0.02


def test_bottom_right_alignment():
    # Sq < Sk: the last Sq rows of the full Sq == Sk problem, with the same positions
    q, k, v = _rand((1, 2, 40, 16), 20), _rand((1, 2, 40, 16), 21), _rand((1, 2, 40, 16), 22)
    full = oracle.rope_attn_fwd(q, k, v, 10000.0, pos_offset=3)
    part = oracle.rope_attn_fwd(q[:, :, 25:], k, v, 10000.0, pos_offset=3)
    np.testing.assert_allclose(part, full[:, :, 25:], atol=1e-13, rtol=0)


def test_rows_subset_matches_full():
    q, k, v = _rand((1, 2, 70, 16), 23), _rand((1, 1, 70, 16), 24), _rand((1, 1, 70, 16), 25)
    full = oracle.rope_attn_fwd(q, k, v, 10000.0)
    rows = np.array([0, 5, 31, 69])
    np.testing.assert_allclose(oracle.rope_attn_fwd(q, k, v, 10000.0, rows=rows),
                               full[:, :, rows], atol=1e-14, rtol=0)


def test_decode_equals_last_prefill_row():
    S = 37
    q, k, v = _rand((2, 4, S, 16), 26), _rand((2, 2, S, 16), 27), _rand((2, 2, S, 16), 28)
    full = oracle.rope_attn_fwd(q, k, v, 10000.0)
    k_cache = oracle.rope_rotate(k, np.arange(S), 10000.0)
    d = oracle.rope_attn_decode(q[:, :, S - 1:], k_cache, v, 10000.0, pos=S - 1)
    np.testing.assert_allclose(d[:, :, 0], full[:, :, S - 1], atol=1e-13, rtol=0)
    # a longer cache with rows past pos is ignored
    pad = np.concatenate([k_cache, _rand((2, 2, 5, 16), 29)], axis=2)
    vpad = np.concatenate([v, _rand((2, 2, 5, 16), 30)], axis=2)
    d2 = oracle.rope_attn_decode(q[:, :, S - 1:], pad, vpad, 10000.0, pos=S - 1)
    np.testing.assert_allclose(d2, d, atol=1e-15, rtol=0)


# ----------------------------------------------------------------- independent brute force

def _brute(q, k, v, base, pos_offset, causal):
    """Scalar loops, math.fsum and math.cos/sin; written separately from the oracle."""
    B, Hq, Sq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, Sk = len(k[0]), len(k[0][0])

    def rot(vec, p):
        out = [0.0] * D
        for i in range(D // 2):
            a = p * base ** (-2.0 * i / D)
            c, s = math.cos(a), math.sin(a)
            out[2 * i] = vec[2 * i] * c - vec[2 * i + 1] * s
            out[2 * i + 1] = vec[2 * i] * s + vec[2 * i + 1] * c
        return out

    res = []
    for b in range(B):
        hb = []
        for h in range(Hq):
            g = h * Hkv // Hq
            rows = []
            for i in range(Sq):
                pi = pos_offset + Sk - Sq + i
                qi = rot(q[b][h][i], pi)
                sc = []
                for j in range(Sk):
                    pj = pos_offset + j
                    if causal and pj > pi:
                        continue
                    kj = rot(k[b][g][j], pj)
                    sc.append((j, math.fsum(x * y for x, y in zip(qi, kj)) / math.sqrt(D)))
                mx = max(s for _, s in sc)
                w = [(j, math.exp(s - mx)) for j, s in sc]
                z = math.fsum(e for _, e in w)
                rows.append([math.fsum(e * v[b][g][j][d] for j, e in w) / z for d in range(D)])
            hb.append(rows)
        res.append(hb)
    return np.array(res)


@pytest.mark.parametrize("Sq,Sk,causal,off", [(8, 8, True, 0), (5, 8, True, 3), (8, 8, False, 0),
                                              (1, 6, True, 9), (7, 3, False, 2)])
def test_brute_force_small(Sq, Sk, causal, off):
    rng = np.random.default_rng(31)
    q = rng.standard_normal((1, 4, Sq, 6))
    k = rng.standard_normal((1, 2, Sk, 6))
    v = rng.standard_normal((1, 2, Sk, 6))
    want = _brute(q.tolist(), k.tolist(), v.tolist(), 10000.0, off, causal)
    got = oracle.rope_attn_fwd(q, k, v, 10000.0, pos_offset=off, causal=causal)
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


def test_torch_sdpa_crosscheck():
    # library cross-check: torch's CPU fp64 SDPA on independently rotated Q/K (complex form)
    q, k, v = (to_f64(t) for t in make_inputs(TINY, seed=0))
    D, S, base = TINY.D, TINY.Sq, TINY.rope_base
    theta = np.array([base ** (-2.0 * i / D) for i in range(D // 2)])
    rot = lambda x: (lambda z: np.stack([z.real, z.imag], -1).reshape(x.shape))(
        (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * np.arange(S)[:, None] * theta))
    qt, kt, vt = (torch.from_numpy(a) for a in (rot(q), rot(k), v))
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True).numpy()
    got = oracle.rope_attn_fwd(q, k, v, base)
    np.testing.assert_allclose(got, want, atol=1e-10, rtol=0)


# ----------------------------------------------------------------- planted mistakes

def test_planted_mistakes_are_caught(monkeypatch):
    """Plant typical mistakes in the oracle (CPU) and check that some pin fails."""
    g3 = read_golden("problem3_rope_relative.txt")

    def sign_pin():
        qr = ref.rope_rotate(np.array([[1.0, 0.0]]), np.array([1]), 10000.0)
        kr = ref.rope_rotate(np.array([[0.0, 1.0]]), np.array([0]), 10000.0)
        return abs(float(qr[0] @ kr[0]) - g3["value"]) < g3["tol"]

    def problem1_pin():
        g = read_golden("problem1_scaled_softmax.txt")
        return np.allclose(_weights_of_one_query(g["logits"], 64), g["scaled_weights"], atol=1e-5)

    def causal_pin():
        q, k, v = _rand((1, 1, 9, 4), 40), _rand((1, 1, 9, 4), 41), _rand((1, 1, 9, 4), 42)
        o = ref.rope_attn_fwd(q, k, v, 10000.0)
        return np.allclose(o[:, :, 0], v[:, :, 0], atol=1e-14)

    assert sign_pin() and problem1_pin() and causal_pin()

    orig_rot = ref.rope_rotate

    def wrong_sense(x, positions, base):
        return orig_rot(x, -np.asarray(positions), base)
    monkeypatch.setattr(ref, "rope_rotate", wrong_sense)
    assert not sign_pin()
    monkeypatch.setattr(ref, "rope_rotate", orig_rot)

    orig_sm = ref._softmax_rows
    monkeypatch.setattr(ref, "_softmax_rows", lambda s: orig_sm(s * math.sqrt(64)))  # scale dropped
    assert not problem1_pin()
    monkeypatch.setattr(ref, "_softmax_rows", orig_sm)

    orig_attn = ref.attention

    def no_mask(q, k, v, causal, rows=None, row_block=1024, window=0):
        return orig_attn(q, k, v, False, rows, row_block, window)
    monkeypatch.setattr(ref, "attention", no_mask)
    assert not causal_pin()
    monkeypatch.setattr(ref, "attention", orig_attn)

    def window_pin():
        q, k, v = _rand((1, 1, 12, 4), 43), _rand((1, 1, 12, 4), 44), _rand((1, 1, 12, 4), 45)
        return np.allclose(ref.rope_attn_fwd(q, k, v, 10000.0, window=1), v, atol=1e-14)

    assert window_pin()

    def window_off_by_one(q, k, v, causal, rows=None, row_block=1024, window=0):
        return orig_attn(q, k, v, causal, rows, row_block, window + 1 if window else 0)
    monkeypatch.setattr(ref, "attention", window_off_by_one)
    assert not window_pin()


# ----------------------------------------------------------------- sliding window

def test_window_one_attends_only_itself():
    # W = 1: each query sees only the key at its own position, so O[i] = V[i + Sk - Sq]
    q, k, v = _rand((1, 2, 20, 8), 50), _rand((1, 2, 30, 8), 51), _rand((1, 2, 30, 8), 52)
    o = oracle.rope_attn_fwd(q, k, v, 10000.0, causal=True, window=1)
    np.testing.assert_allclose(o, v[:, :, 10:], atol=1e-14, rtol=0)


def test_window_covering_everything_is_causal():
    q, k, v = _rand((1, 2, 40, 8), 53), _rand((1, 2, 40, 8), 54), _rand((1, 2, 40, 8), 55)
    np.testing.assert_allclose(oracle.rope_attn_fwd(q, k, v, 10000.0, window=40),
                               oracle.rope_attn_fwd(q, k, v, 10000.0), atol=1e-14, rtol=0)


def test_window_row_equals_causal_on_its_last_keys():
    # row i with window W is plain attention of that query over keys i-W+1 .. i (RoPE is
    # relative, so dropping the older keys and re-basing positions changes nothing)
    S, W = 50, 7
    q, k, v = _rand((1, 1, S, 8), 56), _rand((1, 1, S, 8), 57), _rand((1, 1, S, 8), 58)
    o = oracle.rope_attn_fwd(q, k, v, 10000.0, window=W)
    for i in (0, 3, 6, 7, 31, 49):
        lo = max(0, i - W + 1)
        sub = oracle.rope_attn_fwd(q[:, :, i:i + 1], k[:, :, lo:i + 1], v[:, :, lo:i + 1], 10000.0,
                                   pos_offset=lo)
        np.testing.assert_allclose(o[:, :, i], sub[:, :, 0], atol=1e-12, rtol=0)


def test_window_decode_equals_last_prefill_row():
    S, W = 45, 9
    q, k, v = _rand((1, 4, S, 8), 59), _rand((1, 2, S, 8), 60), _rand((1, 2, S, 8), 61)
    full = oracle.rope_attn_fwd(q, k, v, 10000.0, window=W)
    kc = oracle.rope_rotate(k, np.arange(S), 10000.0)
    d = oracle.rope_attn_decode(q[:, :, S - 1:], kc, v, 10000.0, pos=S - 1, window=W)
    np.testing.assert_allclose(d[:, :, 0], full[:, :, S - 1], atol=1e-13, rtol=0)


def test_brute_force_window():
    # scalar brute force with an explicit window test, written separately from the oracle
    rng = np.random.default_rng(62)
    Sq, Sk, W, D, off = 6, 9, 3, 4, 5
    q, k, v = rng.standard_normal((1, 2, Sq, D)), rng.standard_normal((1, 1, Sk, D)), rng.standard_normal((1, 1, Sk, D))
    want = np.zeros((1, 2, Sq, D))
    for h in range(2):
        for i in range(Sq):
            pi = off + Sk - Sq + i
            def rot(x, p):
                out = np.zeros(D)
                for t in range(D // 2):
                    a = p * 10000.0 ** (-2.0 * t / D)
                    out[2 * t] = x[2 * t] * math.cos(a) - x[2 * t + 1] * math.sin(a)
                    out[2 * t + 1] = x[2 * t] * math.sin(a) + x[2 * t + 1] * math.cos(a)
                return out
            qi = rot(q[0, h, i], pi)
            sc = [(j, float(qi @ rot(k[0, 0, j], off + j)) / math.sqrt(D)) for j in range(Sk)
                  if pi - W < off + j <= pi]
            mx = max(s for _, s in sc)
            e = [(j, math.exp(s - mx)) for j, s in sc]
            z = math.fsum(w for _, w in e)
            want[0, h, i] = sum(w * v[0, 0, j] for j, w in e) / z
    got = oracle.rope_attn_fwd(q, k, v, 10000.0, pos_offset=off, window=W)
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


# ----------------------------------------------------------------- KV-cache flow

def _kv_seq(seed, B=2, Hq=4, Hkv=2, S=40, D=8):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, Hq, S, D)), r.standard_normal((B, Hkv, S, D)),
            r.standard_normal((B, Hkv, S, D)))


@pytest.mark.parametrize("P,window", [(0, 0), (17, 0), (25, 9), (39, 0)])
def test_chunked_prefill_equals_full_prefill(P, window):
    # prefilling tokens P.. on top of a cache that holds tokens 0..P-1 gives the same rows as
    # one prefill of the whole sequence (and the cache ends up holding all rotated keys)
    q, k, v = _kv_seq(70)
    S, cap = k.shape[2], 48
    full = oracle.rope_attn_fwd(q, k, v, 10000.0, window=window)
    kc = np.full((2, 2, cap, 8), np.nan)
    vc = np.full((2, 2, cap, 8), np.nan)
    kc[:, :, :P] = oracle.rope_rotate(k[:, :, :P], np.arange(P), 10000.0)
    vc[:, :, :P] = v[:, :, :P]
    out, kc2, vc2 = oracle.rope_attn_prefill_cached(q[:, :, P:], k[:, :, P:], v[:, :, P:], kc, vc,
                                                    10000.0, P, window=window)
    np.testing.assert_allclose(out, full[:, :, P:], atol=1e-12, rtol=0)
    np.testing.assert_allclose(kc2[:, :, :S], oracle.rope_rotate(k, np.arange(S), 10000.0),
                               atol=1e-14, rtol=0)
    np.testing.assert_array_equal(vc2[:, :, :S], v)
    assert np.isnan(kc2[:, :, S:]).all() and np.isnan(vc2[:, :, S:]).all()  # rows past T untouched


def test_token_by_token_decode_equals_prefill():
    # decoding the sequence one token at a time from an empty cache (each step appends its
    # own key/value at pos) reproduces every row of the causal prefill
    q, k, v = _kv_seq(71, S=24)
    S = k.shape[2]
    full = oracle.rope_attn_fwd(q, k, v, 10000.0)
    kc = np.full((2, 2, 32, 8), np.nan)
    vc = np.full((2, 2, 32, 8), np.nan)
    for p in range(S):
        out, kc, vc = oracle.rope_attn_decode_step(q[:, :, p:p + 1], k[:, :, p:p + 1],
                                                   v[:, :, p:p + 1], kc, vc, 10000.0, [p, p])
        np.testing.assert_allclose(out[:, :, 0], full[:, :, p], atol=1e-12, rtol=0)


def test_varlen_decode_each_sequence_at_its_position():
    q, k, v = _kv_seq(72, B=3, S=30)
    pos = [29, 4, 17]
    kc = oracle.rope_rotate(k, np.arange(30), 10000.0)
    vc = v.copy()
    for window in (0, 6):
        full = oracle.rope_attn_fwd(q, k, v, 10000.0, window=window)
        qd = np.stack([q[b, :, pos[b]] for b in range(3)])[:, :, None]
        # the new tokens are the keys already at pos[b]: appending them again is a no-op
        kn = np.stack([k[b, :, pos[b]] for b in range(3)])[:, :, None]
        vn = np.stack([v[b, :, pos[b]] for b in range(3)])[:, :, None]
        out, kc2, vc2 = oracle.rope_attn_decode_step(qd, kn, vn, kc, vc, 10000.0, pos, window)
        for b in range(3):
            np.testing.assert_allclose(out[b, :, 0], full[b, :, pos[b]], atol=1e-12, rtol=0)
        np.testing.assert_allclose(kc2, kc, atol=1e-14, rtol=0)


def test_gather_pages_by_hand():
    # page 2, blocks [3, 0, 2]: rows 0..5 are block 3 rows 0,1, block 0 rows 0,1, block 2 rows 0,1
    pool = np.zeros((4, 1, 2, 1))
    for blk in range(4):
        for off in range(2):
            pool[blk, 0, off, 0] = 100 * blk + off
    g = oracle.gather_pages(pool, np.array([[3, 0, 2]]), 0, 6)
    assert g[0, :, 0].tolist() == [300, 301, 0, 1, 200, 201]


def test_paged_decode_equals_contiguous():
    rng = np.random.default_rng(73)
    B, Hq, Hkv, D, page, nblk = 3, 4, 2, 8, 4, 9
    pos = [10, 3, 7]
    q = rng.standard_normal((B, Hq, 1, D))
    kn, vn = rng.standard_normal((B, Hkv, 1, D)), rng.standard_normal((B, Hkv, 1, D))
    kc, vc = rng.standard_normal((B, Hkv, 12, D)), rng.standard_normal((B, Hkv, 12, D))
    # scatter each sequence's 12 rows over 3 pages of a shuffled pool
    perm = rng.permutation(nblk)
    table = perm.reshape(B, 3)
    kp = np.full((nblk, Hkv, page, D), np.nan)
    vp = np.full((nblk, Hkv, page, D), np.nan)
    for b in range(B):
        for j in range(12):
            kp[table[b, j // page], :, j % page] = kc[b, :, j]
            vp[table[b, j // page], :, j % page] = vc[b, :, j]
    for window in (0, 5):
        want, kc2, _ = oracle.rope_attn_decode_step(q, kn, vn, kc, vc, 10000.0, pos, window)
        got, kp2, _ = oracle.rope_attn_decode_paged(q, kn, vn, kp, vp, table, 10000.0, pos, window)
        np.testing.assert_array_equal(got, want)
        for b in range(B):
            np.testing.assert_array_equal(oracle.gather_pages(kp2, table, b, 12), kc2[b])


# ----------------------------------------------------------------- ring attention (§6.6)

def _rot_brute(vec, p, base):
    D = len(vec)
    out = [0.0] * D
    for i in range(D // 2):
        a = p * base ** (-2.0 * i / D)
        c, s = math.cos(a), math.sin(a)
        out[2 * i] = vec[2 * i] * c - vec[2 * i + 1] * s
        out[2 * i + 1] = vec[2 * i] * s + vec[2 * i + 1] * c
    return out


def _partial_brute(q, k, v, base, q_pos0, k_pos0, causal):
    """Scalar loops and math.fsum: output and natural-log LSE of one block, with keys
    rotated here at k_pos0 + j. Rows with no allowed key give (zeros, -inf)."""
    B, Hq, Sq, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, Sk = len(k[0]), len(k[0][0])
    o = np.zeros((B, Hq, Sq, D))
    lse = np.full((B, Hq, Sq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h * Hkv // Hq
            for i in range(Sq):
                qi = _rot_brute(q[b][h][i], q_pos0 + i, base)
                sc = []
                for j in range(Sk):
                    if causal and k_pos0 + j > q_pos0 + i:
                        continue
                    kj = _rot_brute(k[b][g][j], k_pos0 + j, base)
                    sc.append((j, math.fsum(x * y for x, y in zip(qi, kj)) / math.sqrt(D)))
                if not sc:
                    continue
                mx = max(s for _, s in sc)
                w = [(j, math.exp(s - mx)) for j, s in sc]
                z = math.fsum(e for _, e in w)
                lse[b, h, i] = mx + math.log(z)
                for d in range(D):
                    o[b, h, i, d] = math.fsum(e * v[b][g][j][d] for j, e in w) / z
    return o, lse


def _rot_keys_brute(k, k_pos0, base):
    return np.array([[[_rot_brute(row, k_pos0 + j, base) for j, row in enumerate(head)]
                      for head in batch] for batch in k.tolist()])


@pytest.mark.parametrize("Sq,Sk,q_pos0,k_pos0,causal", [
    (6, 6, 0, 0, True),      # the diagonal block of a ring
    (5, 7, 9, 0, True),      # a block wholly in the past: every key allowed
    (6, 8, 4, 2, True),      # a block straddling the diagonal
    (4, 6, 1, 3, True),      # the first two rows have no allowed key
    (5, 3, 2, 11, False),    # no mask
])
def test_partial_block_brute_force(Sq, Sk, q_pos0, k_pos0, causal):
    rng = np.random.default_rng(81)
    q = rng.standard_normal((1, 4, Sq, 6))
    k = rng.standard_normal((1, 2, Sk, 6))
    v = rng.standard_normal((1, 2, Sk, 6))
    base = 500.0
    want_o, want_l = _partial_brute(q.tolist(), k.tolist(), v.tolist(), base, q_pos0, k_pos0,
                                    causal)
    k_rot = _rot_keys_brute(k, k_pos0, base)
    got_o, got_l = oracle.rope_attn_fwd_partial(q, k_rot, v, base, q_pos0, k_pos0, causal)
    np.testing.assert_allclose(got_o, want_o, atol=1e-12, rtol=0)
    np.testing.assert_array_equal(np.isfinite(got_l), np.isfinite(want_l))
    fin = np.isfinite(want_l)
    np.testing.assert_allclose(got_l[fin], want_l[fin], atol=1e-12, rtol=0)


def test_partial_single_key_lse_is_the_score():
    # one key at the query's own position: the rotation cancels, LSE = q.k / sqrt(D)
    rng = np.random.default_rng(82)
    q, k, v = rng.standard_normal((1, 1, 1, 8)), rng.standard_normal((1, 1, 1, 8)), \
        rng.standard_normal((1, 1, 1, 8))
    k_rot = ref.rope_rotate(k, np.array([5]), 10000.0)
    o, lse = oracle.rope_attn_fwd_partial(q, k_rot, v, 10000.0, 5, 5, True)
    np.testing.assert_allclose(lse[0, 0, 0], float(q[0, 0, 0] @ k[0, 0, 0]) / math.sqrt(8),
                               atol=1e-13, rtol=0)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-14, rtol=0)


@pytest.mark.parametrize("causal", [True, False])
def test_merge_of_key_splits_equals_whole_block(causal):
    rng = np.random.default_rng(83)
    Sq, Sk, q_pos0 = 9, 13, 6
    q = rng.standard_normal((2, 4, Sq, 8))
    k_rot = ref.rope_rotate(rng.standard_normal((2, 2, Sk, 8)), np.arange(Sk), 10000.0)
    v = rng.standard_normal((2, 2, Sk, 8))
    whole_o, whole_l = oracle.rope_attn_fwd_partial(q, k_rot, v, 10000.0, q_pos0, 0, causal)
    for a in (1, 5, 12):
        o1, l1 = oracle.rope_attn_fwd_partial(q, k_rot[:, :, :a], v[:, :, :a], 10000.0, q_pos0,
                                              0, causal)
        o2, l2 = oracle.rope_attn_fwd_partial(q, k_rot[:, :, a:], v[:, :, a:], 10000.0, q_pos0,
                                              a, causal)
        for mo, ml in (oracle.merge_partials(o1, l1, o2, l2), oracle.merge_partials(o2, l2, o1, l1)):
            np.testing.assert_allclose(mo, whole_o, atol=1e-13, rtol=0)
            np.testing.assert_allclose(ml, whole_l, atol=1e-13, rtol=0)


def test_merge_with_an_empty_partial_is_identity():
    rng = np.random.default_rng(84)
    o, lse = rng.standard_normal((1, 2, 5, 4)), rng.standard_normal((1, 2, 5))
    empty_o, empty_l = np.zeros_like(o), np.full_like(lse, -np.inf)
    for mo, ml in (oracle.merge_partials(o, lse, empty_o, empty_l),
                   oracle.merge_partials(empty_o, empty_l, o, lse)):
        np.testing.assert_allclose(mo, o, atol=1e-15, rtol=0)
        np.testing.assert_allclose(ml, lse, atol=1e-15, rtol=0)
    mo, ml = oracle.merge_partials(empty_o, empty_l, empty_o, empty_l)
    assert np.all(mo == 0) and np.all(ml == -np.inf)


def test_ring_shards_cover_the_sequence():
    for S, n in ((64, 4), (37, 3), (5, 5), (7, 2)):
        sh = oracle.ring_shards(S, n)
        assert sh[0][0] == 0 and sh[-1][1] == S and len(sh) == n
        assert all(a[1] == b[0] for a, b in zip(sh, sh[1:]))
        assert max(b - a for a, b in sh) - min(b - a for a, b in sh) <= 1


@pytest.mark.parametrize("S,n", [(37, 1), (37, 2), (37, 3), (64, 4), (30, 5)])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_equals_full_attention(S, n, causal):
    rng = np.random.default_rng(85)
    q = rng.standard_normal((2, 4, S, 8))
    k = rng.standard_normal((2, 2, S, 8))
    v = rng.standard_normal((2, 2, S, 8))
    o, lse = oracle.ring_attention(q, k, v, 10000.0, n, causal)
    np.testing.assert_allclose(o, oracle.rope_attn_fwd(q, k, v, 10000.0, 0, causal),
                               atol=1e-13, rtol=0)
    k_rot = ref.rope_rotate(k, np.arange(S), 10000.0)
    _, whole_l = oracle.rope_attn_fwd_partial(q, k_rot, v, 10000.0, 0, 0, causal)
    np.testing.assert_allclose(lse, whole_l, atol=1e-13, rtol=0)


def test_ring_diagonal_block_is_prefill_at_its_offset():
    rng = np.random.default_rng(86)
    a, L = 21, 11
    q, k, v = rng.standard_normal((1, 4, L, 8)), rng.standard_normal((1, 2, L, 8)), \
        rng.standard_normal((1, 2, L, 8))
    k_rot = ref.rope_rotate(k, a + np.arange(L), 10000.0)
    o, _ = oracle.rope_attn_fwd_partial(q, k_rot, v, 10000.0, a, a, True)
    np.testing.assert_allclose(o, oracle.rope_attn_fwd(q, k, v, 10000.0, pos_offset=a),
                               atol=1e-13, rtol=0)


def test_planted_ring_mistakes_are_caught(monkeypatch):
    rng = np.random.default_rng(87)
    q, k, v = rng.standard_normal((1, 2, 24, 4)), rng.standard_normal((1, 1, 24, 4)), \
        rng.standard_normal((1, 1, 24, 4))
    full = oracle.rope_attn_fwd(q, k, v, 10000.0)

    def ring_pin():
        return np.allclose(ref.ring_attention(q, k, v, 10000.0, 3)[0], full, atol=1e-12)

    def lse_pin():
        o, l = ref.rope_attn_fwd_partial(q[:, :, :3], ref.rope_rotate(k[:, :, :3], np.arange(3),
                                                                      10000.0),
                                         v[:, :, :3], 10000.0, 0, 0, True)
        want_o, want_l = _partial_brute(q[:, :, :3].tolist(), k[:, :, :3].tolist(),
                                        v[:, :, :3].tolist(), 10000.0, 0, 0, True)
        return np.allclose(l, want_l, atol=1e-12)

    assert ring_pin() and lse_pin()
    orig_merge, orig_partial = ref.merge_partials, ref.rope_attn_fwd_partial

    # weights of the two sides swapped
    monkeypatch.setattr(ref, "merge_partials",
                        lambda oa, la, ob, lb: (orig_merge(oa, lb, ob, la)[0],
                                                orig_merge(oa, la, ob, lb)[1]))
    assert not ring_pin()
    monkeypatch.setattr(ref, "merge_partials", orig_merge)

    # key positions off by one inside a block
    monkeypatch.setattr(ref, "rope_attn_fwd_partial",
                        lambda q_, k_, v_, b_, qp, kp, c_=True: orig_partial(q_, k_, v_, b_, qp,
                                                                              kp + 1, c_))
    assert not ring_pin()
    monkeypatch.setattr(ref, "rope_attn_fwd_partial", orig_partial)

    # the causal mask dropped inside blocks
    monkeypatch.setattr(ref, "rope_attn_fwd_partial",
                        lambda q_, k_, v_, b_, qp, kp, c_=True: orig_partial(q_, k_, v_, b_, qp,
                                                                              kp, False))
    assert not ring_pin()
    monkeypatch.setattr(ref, "rope_attn_fwd_partial", orig_partial)

    # the LSE without the row max (log of the shifted sum only)
    def lse_without_max(q_, k_, v_, b_, qp, kp, c_=True):
        o, l = orig_partial(q_, k_, v_, b_, qp, kp, c_)
        D = q_.shape[-1]
        qr = ref.rope_rotate(q_, qp + np.arange(q_.shape[2]), b_)
        s = np.einsum("bhid,bhjd->bhij", qr, np.repeat(k_, q_.shape[1] // k_.shape[1], 1))
        return o, l - np.max(s, axis=-1) / math.sqrt(D)
    monkeypatch.setattr(ref, "rope_attn_fwd_partial", lse_without_max)
    assert not lse_pin()


def test_zigzag_chunks_cover_the_sequence_once():
    for S, n in ((32, 4), (12, 3), (4, 2), (16, 1)):
        ch = oracle.zigzag_chunks(S, n)
        spans = sorted(rng for pair in ch for rng in pair)
        assert spans[0][0] == 0 and spans[-1][1] == S
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        # each rank's two chunks are mirror images: their causal work is the same for all ranks
        assert all(lo[0] + hi[0] == S - (S // (2 * n)) for lo, hi in ch)


@pytest.mark.parametrize("S,n", [(40, 1), (40, 2), (36, 3), (64, 4)])
@pytest.mark.parametrize("causal", [True, False])
def test_zigzag_ring_equals_full_attention(S, n, causal):
    rng = np.random.default_rng(88)
    q = rng.standard_normal((2, 4, S, 8))
    k = rng.standard_normal((2, 2, S, 8))
    v = rng.standard_normal((2, 2, S, 8))
    o, lse = oracle.ring_attention_zigzag(q, k, v, 10000.0, n, causal)
    np.testing.assert_allclose(o, oracle.rope_attn_fwd(q, k, v, 10000.0, 0, causal),
                               atol=1e-13, rtol=0)
    _, want_l = oracle.ring_attention(q, k, v, 10000.0, 1, causal)
    np.testing.assert_allclose(lse, want_l, atol=1e-13, rtol=0)


def test_planted_zigzag_mistakes_are_caught(monkeypatch):
    rng = np.random.default_rng(89)
    q, k, v = rng.standard_normal((1, 2, 24, 4)), rng.standard_normal((1, 1, 24, 4)), \
        rng.standard_normal((1, 1, 24, 4))
    full = oracle.rope_attn_fwd(q, k, v, 10000.0)

    def pin():
        return np.allclose(ref.ring_attention_zigzag(q, k, v, 10000.0, 3)[0], full, atol=1e-12)

    assert pin()
    orig = ref.zigzag_chunks
    # a rank's second chunk taken at the wrong place (2n-2-r instead of 2n-1-r), so one chunk
    # is never a key and another is used twice
    monkeypatch.setattr(ref, "zigzag_chunks", lambda S, n: [
        (a, ((2 * n - 2 - r) * (S // (2 * n)), (2 * n - 1 - r) * (S // (2 * n))))
        for r, (a, _) in enumerate(orig(S, n))])
    assert not pin()


def test_merge_is_associative_and_commutative():
    # three partials over disjoint key ranges combine to the same result in any grouping/order
    rng = np.random.default_rng(90)
    q = rng.standard_normal((1, 2, 5, 8))
    k_rot = ref.rope_rotate(rng.standard_normal((1, 1, 30, 8)), np.arange(30), 10000.0)
    v = rng.standard_normal((1, 1, 30, 8))
    parts = [oracle.rope_attn_fwd_partial(q, k_rot[:, :, a:b], v[:, :, a:b], 10000.0, 40, a, True)
             for a, b in ((0, 7), (7, 19), (19, 30))]
    m = oracle.merge_partials
    left = m(*m(*parts[0], *parts[1]), *parts[2])
    right = m(*parts[0], *m(*parts[1], *parts[2]))
    swapped = m(*m(*parts[2], *parts[0]), *parts[1])
    whole = oracle.rope_attn_fwd_partial(q, k_rot, v, 10000.0, 40, 0, True)
    for o, lse in (left, right, swapped):
        np.testing.assert_allclose(o, whole[0], atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse, whole[1], atol=1e-13, rtol=0)
