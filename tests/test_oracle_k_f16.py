"""Pins of the oracle with K stored as f16 (the f16-f16 pair, which the
flash-attention build always compiles: "llama.cpp adaptive KV streaming - spec
fork notes", TLDR).  The K "blocks" are the fp16 values themselves, so the
scores are the exact dot products with those values, and with f16 V too the
oracle is the exact attention over the inputs."""
import math

import numpy as np
from scipy.special import logsumexp, softmax

import oracle

D = 128
KF = oracle.K_F16
VF = oracle.V_F16


def test_k_blocks_are_the_input_bits():
    rng = np.random.default_rng(211)
    k = (rng.standard_normal((5, 3, D)) * 50).astype(np.float16)
    v = rng.standard_normal((5, 3, D)).astype(np.float16)
    k[1, 2, :4] = np.array([0.0, -0.0, -65504.0, 2.0 ** -24], np.float16)  # zero signs, extremes
    kb, vb = oracle.quantize_rows(k, v, v_type=VF, k_type=KF)
    assert kb.shape == (5, 3, 4, 64) and vb.shape == (5, 3, 4, 64)
    assert np.array_equal(kb.reshape(5, 3, D * 2).view(np.uint16), k.view(np.uint16))
    assert np.array_equal(vb.reshape(5, 3, D * 2).view(np.uint16), v.view(np.uint16))
    # V blocks do not depend on the K type
    _, vq = oracle.quantize_rows(k, v, v_type=oracle.V_Q4_0, k_type=KF)
    _, vq8 = oracle.quantize_rows(k, v, v_type=oracle.V_Q4_0)
    assert np.array_equal(vq, vq8)


def test_f16_f16_against_scipy_over_exact_values():
    rng = np.random.default_rng(212)
    n_keys, n_kv, n_qh, n_q = 140, 2, 8, 3
    k = rng.standard_normal((n_keys, n_kv, D)).astype(np.float16)
    v = rng.standard_normal((n_keys, n_kv, D)).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v, v_type=VF, k_type=KF)
    q = rng.standard_normal((n_q, n_qh, D)).astype(np.float16)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, q, pos0, v_type=VF, k_type=KF)
    G = n_qh // n_kv
    for j in range(n_q):
        for hq in range(n_qh):
            g = hq // G
            nv = pos0 + j + 1
            s = k[:nv, g].astype(np.float64) @ q[j, hq].astype(np.float64) / math.sqrt(D)
            np.testing.assert_allclose(out[j, hq], softmax(s) @ v[:nv, g].astype(np.float64), rtol=0, atol=1e-12)
            assert abs(lse[j, hq] - logsumexp(s)) < 1e-12


def test_f16_k_with_a_dominant_key_selects_its_value():
    rng = np.random.default_rng(213)
    n_keys = 40
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    k = (rng.standard_normal((n_keys, 1, D)) * 0.01).astype(np.float16)
    k[17, 0] = (q[0, 0].astype(np.float32) * 8).astype(np.float16)  # score about 8 |q|^2 / sqrt(128)
    v = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v, v_type=VF, k_type=KF)
    out, _ = oracle.attention(kb, vb, q, n_keys - 1, v_type=VF, k_type=KF)
    np.testing.assert_allclose(out[0, 0], v[17, 0].astype(np.float64), rtol=0, atol=1e-9)
