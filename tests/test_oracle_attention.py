"""Pins of the oracle's attention against closed forms and library routines.

Each case is chosen so that a plausible slip (wrong GQA mapping, off-by-one in
the causal length, a missing or wrong 1/sqrt(d) scale, a transposed operand, a
dropped normalisation, natural vs base-2 log) fails at least one of them.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle

D = 128


def quant(k, v):
    return oracle.quantize_rows(k.astype(np.float16), v.astype(np.float16))


def deq_v(vb):
    """dequantized V [n_keys, n_kv, D] from oracle blocks (dequant itself is pinned)."""
    n, g, nb, _ = vb.shape
    out = np.zeros((n, g, D))
    for i in range(n):
        for j in range(g):
            out[i, j] = np.concatenate([oracle.dequant_q4_0(vb[i, j, b].tobytes()) for b in range(nb)])
    return out


def deq_k(kb):
    n, g, nb, _ = kb.shape
    out = np.zeros((n, g, D))
    for i in range(n):
        for j in range(g):
            out[i, j] = np.concatenate([oracle.dequant_q8_0(kb[i, j, b].tobytes()) for b in range(nb)])
    return out


def test_zero_query_is_uniform_mean_with_causal_lengths():
    # q = 0 -> all scores 0 -> o = mean of the visible values, lse = ln(#visible)
    rng = np.random.default_rng(1)
    n_keys, n_kv, n_qh, n_q = 37, 2, 4, 3
    k = rng.standard_normal((n_keys, n_kv, D))
    v = rng.standard_normal((n_keys, n_kv, D))
    kb, vb = quant(k, v)
    vd = deq_v(vb)
    pos0 = n_keys - n_q
    q = np.zeros((n_q, n_qh, D), np.float16)
    out, lse = oracle.attention(kb, vb, q, pos0)
    for j in range(n_q):
        n_vis = pos0 + j + 1
        for hq in range(n_qh):
            g = hq // (n_qh // n_kv)
            np.testing.assert_allclose(out[j, hq], vd[:n_vis, g].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[j, hq] - math.log(n_vis)) < 1e-13


def test_gqa_grouping_is_contiguous():
    # kv head g holds the constant value (g+1)/8 in every V element: q head h must read g = h // G
    n_keys, n_kv, n_qh = 5, 4, 12
    rng = np.random.default_rng(2)
    k = rng.standard_normal((n_keys, n_kv, D))
    v = np.zeros((n_keys, n_kv, D))
    for g in range(n_kv):
        v[:, g, :] = (g + 1) / 8.0
    kb, vb = quant(k, v)
    q = rng.standard_normal((1, n_qh, D)).astype(np.float16)
    out, _ = oracle.attention(kb, vb, q, n_keys - 1)
    G = n_qh // n_kv
    for hq in range(n_qh):
        np.testing.assert_allclose(out[0, hq], (hq // G + 1) / 8.0, rtol=0, atol=1e-14)


def test_identical_keys_give_mean_and_log_count():
    rng = np.random.default_rng(3)
    n_keys = 64
    krow = rng.standard_normal(D)
    k = np.tile(krow, (n_keys, 1, 1))
    v = rng.standard_normal((n_keys, 1, D))
    kb, vb = quant(k, v)
    kd = deq_k(kb)[0, 0]
    vd = deq_v(vb)
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    out, lse = oracle.attention(kb, vb, q, n_keys - 1)
    np.testing.assert_allclose(out[0, 0], vd[:, 0].mean(axis=0), rtol=0, atol=1e-12)
    s = float(np.dot(q[0, 0].astype(np.float64), kd)) / math.sqrt(D)
    assert abs(lse[0, 0] - (s + math.log(n_keys))) < 1e-12


def test_dominant_key_is_one_hot():
    rng = np.random.default_rng(4)
    n_keys = 50
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    qd = q[0, 0].astype(np.float64)
    k = rng.standard_normal((n_keys, 1, D)) * 0.01
    hot = 17
    k[hot, 0] = 1000.0 * qd / np.linalg.norm(qd)  # |s_hot| ~ 1000*|q|/sqrt(128) >> others
    v = rng.standard_normal((n_keys, 1, D))
    kb, vb = quant(k, v)
    vd = deq_v(vb)
    out, _ = oracle.attention(kb, vb, q, n_keys - 1)
    np.testing.assert_allclose(out[0, 0], vd[hot, 0], rtol=0, atol=1e-12)


def test_two_key_closed_form_pins_scale():
    # q = c e_0, k_0 = a e_0, k_1 = 0: s_0 = c * khat_0 / sqrt(128), s_1 = 0
    c, a = 3.0, 7.9375  # a = 127/16: d = a/127 = 1/16 is exact in fp16
    q = np.zeros((1, 1, D), np.float16)
    q[0, 0, 0] = c
    k = np.zeros((2, 1, D))
    k[0, 0, 0] = a
    rng = np.random.default_rng(5)
    v = rng.standard_normal((2, 1, D))
    kb, vb = quant(k, v)
    khat = oracle.dequant_q8_0(kb[0, 0, 0].tobytes())[0]
    assert khat == a  # a single non-zero value reconstructs exactly when a/127 is an fp16 value
    vd = deq_v(vb)
    s0 = c * khat / math.sqrt(128.0)
    w0 = math.exp(s0) / (math.exp(s0) + 1.0)
    out, lse = oracle.attention(kb, vb, q, 1)
    np.testing.assert_allclose(out[0, 0], w0 * vd[0, 0] + (1 - w0) * vd[1, 0], rtol=0, atol=1e-14)
    assert abs(lse[0, 0] - math.log(math.exp(s0) + 1.0)) < 1e-14


def test_single_key_returns_its_value():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((1, 1, D))
    v = rng.standard_normal((1, 1, D))
    kb, vb = quant(k, v)
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    out, lse = oracle.attention(kb, vb, q, 0)
    np.testing.assert_array_equal(out[0, 0], deq_v(vb)[0, 0])
    s = float(np.dot(q[0, 0].astype(np.float64), deq_k(kb)[0, 0])) / math.sqrt(D)
    assert abs(lse[0, 0] - s) < 1e-13


def test_against_scipy_softmax_random():
    # library softmax / logsumexp over numpy matmuls of the dequantized operands
    rng = np.random.default_rng(7)
    n_keys, n_kv, n_qh, n_q = 300, 2, 6, 4
    k = rng.standard_normal((n_keys, n_kv, D))
    v = rng.standard_normal((n_keys, n_kv, D))
    kb, vb = quant(k, v)
    kd, vd = deq_k(kb), deq_v(vb)
    q = rng.standard_normal((n_q, n_qh, D)).astype(np.float16)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, q, pos0)
    for j in range(n_q):
        for hq in range(n_qh):
            g = hq // (n_qh // n_kv)
            nv = pos0 + j + 1
            s = kd[:nv, g] @ q[j, hq].astype(np.float64) / math.sqrt(D)
            np.testing.assert_allclose(out[j, hq], softmax(s) @ vd[:nv, g], rtol=0, atol=1e-12)
            assert abs(lse[j, hq] - logsumexp(s)) < 1e-12


def test_key_permutation_invariance():
    rng = np.random.default_rng(8)
    n_keys = 40
    k = rng.standard_normal((n_keys, 1, D))
    v = rng.standard_normal((n_keys, 1, D))
    kb, vb = quant(k, v)
    perm = rng.permutation(n_keys)
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    o1, l1 = oracle.attention(kb, vb, q, n_keys - 1)
    o2, l2 = oracle.attention(kb[perm].copy(), vb[perm].copy(), q, n_keys - 1)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_rejects_bad_shapes():
    kb = np.zeros((4, 3, 4, 34), np.uint8)
    vb = np.zeros((4, 3, 4, 18), np.uint8)
    q = np.zeros((1, 4, D), np.float16)  # 4 q heads over 3 kv heads: not a whole group
    with pytest.raises(ValueError):
        oracle.attention(kb, vb, q, 0)
