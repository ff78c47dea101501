"""Pins of the oracle with V stored as f16 (the q8_0-f16 pair, a legal pair of
the flash-attention build list): the V "blocks" are the fp16 values themselves,
and attention over them is the exact attention over those values."""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle

D = 128
F16 = oracle.V_F16


def test_v_blocks_are_the_input_bits():
    rng = np.random.default_rng(111)
    k = rng.standard_normal((7, 2, D)).astype(np.float16)
    v = (rng.standard_normal((7, 2, D)) * 100).astype(np.float16)
    v[0, 0, :4] = np.array([0.0, -0.0, 65504.0, 2.0 ** -24], np.float16)  # zero signs, extremes
    kb, vb = oracle.quantize_rows(k, v, v_type=F16)
    assert vb.shape == (7, 2, 4, 64)
    assert np.array_equal(vb.reshape(7, 2, D * 2).view(np.uint16), v.view(np.uint16))
    kb4, _ = oracle.quantize_rows(k, v)
    assert np.array_equal(kb, kb4)  # K is Q8_0 either way


def test_against_scipy_over_exact_values():
    rng = np.random.default_rng(112)
    n_keys, n_kv, n_qh, n_q = 150, 2, 6, 3
    k = rng.standard_normal((n_keys, n_kv, D)).astype(np.float16)
    v = rng.standard_normal((n_keys, n_kv, D)).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v, v_type=F16)
    kd = np.zeros((n_keys, n_kv, D))
    for i in range(n_keys):
        for g in range(n_kv):
            kd[i, g] = np.concatenate([oracle.dequant_q8_0(kb[i, g, b].tobytes()) for b in range(4)])
    q = rng.standard_normal((n_q, n_qh, D)).astype(np.float16)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, q, pos0, v_type=F16)
    for j in range(n_q):
        for hq in range(n_qh):
            g = hq // 3
            nv = pos0 + j + 1
            s = kd[:nv, g] @ q[j, hq].astype(np.float64) / math.sqrt(D)
            np.testing.assert_allclose(out[j, hq], softmax(s) @ v[:nv, g].astype(np.float64), rtol=0, atol=1e-12)
            assert abs(lse[j, hq] - logsumexp(s)) < 1e-12


def test_zero_query_is_uniform_mean_of_the_values():
    rng = np.random.default_rng(113)
    n_keys, n_q = 33, 2
    k = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    v = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v, v_type=F16)
    out, lse = oracle.attention(kb, vb, np.zeros((n_q, 2, D), np.float16), n_keys - n_q, v_type=F16)
    for j in range(n_q):
        n_vis = n_keys - n_q + j + 1
        for hq in range(2):
            np.testing.assert_allclose(out[j, hq], v[:n_vis, 0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[j, hq] - math.log(n_vis)) < 1e-13


def test_block_size_must_match_the_type():
    with pytest.raises(AssertionError):
        oracle.attention(np.zeros((2, 1, 4, 34), np.uint8), np.zeros((2, 1, 4, 34), np.uint8),
                         np.zeros((1, 1, D), np.float16), 1, v_type=F16)
