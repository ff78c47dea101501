"""Pins of the oracle with V stored as Q8_0 (the q8_0 / q8_0 type pair of the
"Feature/adaptive kv stream integration" pull request's runs): the V blocks are
the pinned Q8_0 block quantizer's, and attention over them matches closed forms
and library routines as with Q4_0 V."""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle

D = 128
Q8 = oracle.V_Q8_0


def quant8(k, v):
    return oracle.quantize_rows(k.astype(np.float16), v.astype(np.float16), v_type=Q8)


def deq(blocks, fn):
    n, g, nb, _ = blocks.shape
    out = np.zeros((n, g, D))
    for i in range(n):
        for j in range(g):
            out[i, j] = np.concatenate([fn(blocks[i, j, b].tobytes()) for b in range(nb)])
    return out


def test_v_blocks_are_the_q8_0_block_quantizer():
    rng = np.random.default_rng(11)
    k = rng.standard_normal((9, 2, D)).astype(np.float16)
    v = (rng.standard_normal((9, 2, D)) * 3).astype(np.float16)
    kb, vb = quant8(k, v)
    assert vb.shape == (9, 2, 4, 34)
    for i in range(9):
        for g in range(2):
            for b in range(4):
                assert vb[i, g, b].tobytes() == oracle.q8_0_block(v[i, g, 32 * b:32 * b + 32])
                assert kb[i, g, b].tobytes() == oracle.q8_0_block(k[i, g, 32 * b:32 * b + 32])
    # the Q4_0 path of the same rows is untouched
    kb4, vb4 = oracle.quantize_rows(k, v)
    assert np.array_equal(kb4, kb) and vb4.shape == (9, 2, 4, 18)


def test_zero_query_is_uniform_mean():
    rng = np.random.default_rng(12)
    n_keys, n_kv, n_qh, n_q = 29, 2, 4, 3
    kb, vb = quant8(rng.standard_normal((n_keys, n_kv, D)), rng.standard_normal((n_keys, n_kv, D)))
    vd = deq(vb, oracle.dequant_q8_0)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, np.zeros((n_q, n_qh, D), np.float16), pos0, v_type=Q8)
    for j in range(n_q):
        n_vis = pos0 + j + 1
        for hq in range(n_qh):
            np.testing.assert_allclose(out[j, hq], vd[:n_vis, hq // 2].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[j, hq] - math.log(n_vis)) < 1e-13


def test_against_scipy_softmax_random():
    rng = np.random.default_rng(13)
    n_keys, n_kv, n_qh, n_q = 200, 2, 6, 3
    kb, vb = quant8(rng.standard_normal((n_keys, n_kv, D)), rng.standard_normal((n_keys, n_kv, D)))
    kd, vd = deq(kb, oracle.dequant_q8_0), deq(vb, oracle.dequant_q8_0)
    q = rng.standard_normal((n_q, n_qh, D)).astype(np.float16)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, q, pos0, v_type=Q8)
    for j in range(n_q):
        for hq in range(n_qh):
            g = hq // 3
            nv = pos0 + j + 1
            s = kd[:nv, g] @ q[j, hq].astype(np.float64) / math.sqrt(D)
            np.testing.assert_allclose(out[j, hq], softmax(s) @ vd[:nv, g], rtol=0, atol=1e-12)
            assert abs(lse[j, hq] - logsumexp(s)) < 1e-12


def test_q8_0_v_is_closer_to_unquantized_values_than_q4_0():
    """Same inputs, same K: only the V quantization differs, and the 8-bit one
    lands much nearer the attention over the exact fp16 values."""
    rng = np.random.default_rng(14)
    n_keys = 120
    k = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    v = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    kb8, vb8 = quant8(k, v)
    kb4, vb4 = oracle.quantize_rows(k, v)
    o8, l8 = oracle.attention(kb8, vb8, q, n_keys - 1, v_type=Q8)
    o4, l4 = oracle.attention(kb4, vb4, q, n_keys - 1)
    assert l8[0, 0] == l4[0, 0]  # scores do not involve V
    kd = deq(kb8, oracle.dequant_q8_0)[:, 0]
    p = softmax(kd @ q[0, 0].astype(np.float64) / math.sqrt(D))
    exact = p @ v[:, 0].astype(np.float64)
    e8, e4 = np.abs(o8[0, 0] - exact).max(), np.abs(o4[0, 0] - exact).max()
    assert e8 < e4 / 8


def test_block_size_must_match_the_type():
    kb = np.zeros((2, 1, 4, 34), np.uint8)
    vb = np.zeros((2, 1, 4, 18), np.uint8)
    with pytest.raises(AssertionError):
        oracle.attention(kb, vb, np.zeros((1, 1, D), np.float16), 1, v_type=Q8)
