"""Pins of the oracle's Q5_0 V blocks (a 5-bit member of the block family the
pages list among the legal cache types; the rule is read as Q4_0's with 32
levels, d = m/-16, q = min(31, trunc(x/d + 16.5))).

* hand-worked blocks (tests/golden/q5_0_hand.txt), including the bit layout;
* brute force: every code is the level nearest x/d, ties to the upper level,
  clamped to 31;
* the per-block error bounds and range invariants the rule implies;
* attention over Q5_0 V: closed forms and library routines, as for Q4_0 V, and
  an error between the Q4_0 and Q8_0 ones on the same inputs.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from golden_io import read_fixture

D = 128
Q5 = oracle.V_Q5_0


def h(vals):
    return np.asarray(vals, np.float64).astype(np.float16)


def split_q5(blk: bytes):
    """(d bits, codes) of a 22-byte block, unpacked independently of the oracle."""
    d = int.from_bytes(blk[:2], "little")
    high = int.from_bytes(blk[2:6], "little")
    b = np.frombuffer(blk[6:], np.uint8).astype(int)
    low = np.concatenate([b & 0xF, b >> 4])
    top = np.array([(high >> i) & 1 for i in range(32)])
    return d, low | (top << 4)


def test_q5_0_hand_worked():
    f, _ = read_fixture("q5_0_hand.txt")
    # D: division, not a rounded reciprocal; E: the binary32 d, not the stored fp16 d
    for tag in ("A", "B", "C", "D", "E"):
        xs = [float(v) for v in f[f"{tag}_x"]]
        x = h(xs)
        assert np.array_equal(x.astype(np.float64), np.array(xs))  # the inputs are exact in fp16
        blk = oracle.q5_0_block(x)
        assert len(blk) == 22
        d, q = split_q5(blk)
        assert d == int(f[f"{tag}_d_bits"][0], 16)
        if f"{tag}_q" in f:
            assert q.tolist() == [int(v) for v in f[f"{tag}_q"]]
        if f"{tag}_bytes" in f:
            assert list(blk[2:]) == [int(v, 16) for v in f[f"{tag}_bytes"]]


def test_q5_0_dequant_of_hand_block():
    """A's reconstruction is d (q - 16) with d = 0.0625: exact values."""
    f, _ = read_fixture("q5_0_hand.txt")
    blk = oracle.q5_0_block(h([float(v) for v in f["A_x"]]))
    q = np.array([int(v) for v in f["A_q"]])
    assert np.array_equal(oracle.dequant_q5_0(blk), 0.0625 * (q - 16))


def _blocks(rng, n):
    for i in range(n):
        kind = i % 4
        if kind == 0:
            x = rng.standard_normal(32)
        elif kind == 1:
            x = rng.uniform(-1, 1, 32) * 10.0 ** rng.integers(-4, 4)
        elif kind == 2:  # many exact ties of the +16.5 rounding
            x = (rng.integers(-32, 33, 32) / 2.0) * 2.0 ** rng.integers(-6, 3)
        else:
            x = rng.standard_normal(32)
            x[rng.integers(0, 32)] *= 40.0
        yield h(x)


def test_q5_0_brute_force_nearest_level():
    """Every code is the level q - 16 nearest to r = x/d (binary32), ties to the
    upper level, clamped to 31, found by trying all 32 codes."""
    rng = np.random.default_rng(31)
    levels = np.arange(32) - 16
    for x in _blocks(rng, 400):
        blk = oracle.q5_0_block(x)
        _, q = split_q5(blk)
        xf = x.astype(np.float32)
        i_max = int(np.argmax(np.abs(xf)))
        d32 = np.float32(xf[i_max]) / np.float32(-16)
        if d32 == 0:
            assert (q == 16).all()
            continue
        for i in range(32):
            r = float(np.float32(xf[i]) / np.float32(d32))
            dist = np.abs(r - levels)
            best = np.flatnonzero(dist == dist.min())
            want = int(best.max())  # upper level on a tie; past the top level, the top one
            assert q[i] == want, (i, r, q[i], want)


def test_q5_0_error_bound_and_range():
    rng = np.random.default_rng(32)
    for x in _blocks(rng, 1500):
        blk = oracle.q5_0_block(x)
        d_bits, q = split_q5(blk)
        xf = x.astype(np.float64)
        i_max = int(np.argmax(np.abs(xf)))
        m = xf[i_max]
        d32 = float(np.float32(np.float32(m) / np.float32(-16)))
        dh = float(np.uint16(d_bits).view(np.float16))
        assert q.min() >= 0 and q.max() <= 31
        deq = oracle.dequant_q5_0(blk)
        assert np.array_equal(deq, dh * (q - 16))
        if d32 == 0:
            continue
        assert q[i_max] == 0 and deq[i_max] == -16 * dh
        ratio = xf / d32
        clamped = ratio > 15.5
        err32 = np.abs(xf - (q - 16) * d32)
        tol = abs(d32) * 2 ** -20
        assert np.all(err32[~clamped] <= abs(d32) / 2 + tol)
        assert np.all(err32[clamped] <= abs(d32) + tol)
        extra = np.abs(q - 16) * abs(dh - d32)
        assert np.all(np.abs(xf - deq) <= err32 + extra + tol)


def test_q5_0_is_twice_as_fine_as_q4_0():
    """Same block: the 32-level grid's step is half the 16-level one's (the
    signed max over -16 against over -8), so its rms error is about half."""
    rng = np.random.default_rng(33)
    se4 = se5 = 0.0
    for _ in range(300):
        x = h(rng.standard_normal(32))
        b4, b5 = oracle.q4_0_block(x), oracle.q5_0_block(x)
        d4 = float(np.frombuffer(b4[:2], np.float16)[0])
        d5 = float(np.frombuffer(b5[:2], np.float16)[0])
        assert abs(d5 - d4 / 2) <= abs(d4) * 2 ** -10
        xf = x.astype(np.float64)
        e5 = oracle.dequant_q5_0(b5) - xf
        assert np.abs(e5).max() <= abs(d5) * (1 + 2 ** -9)  # at most one step (a clamped top value)
        se4 += float(np.sum((oracle.dequant_q4_0(b4) - xf) ** 2))
        se5 += float(np.sum(e5 ** 2))
    assert 0.4 < math.sqrt(se5 / se4) < 0.6


def test_quantize_rows_q5_0_matches_blocks():
    rng = np.random.default_rng(34)
    k = rng.standard_normal((5, 2, D)).astype(np.float16)
    v = (rng.standard_normal((5, 2, D)) * 2).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v, v_type=Q5)
    assert kb.shape == (5, 2, 4, 34) and vb.shape == (5, 2, 4, 22)
    for t in range(5):
        for g in range(2):
            for b in range(4):
                assert vb[t, g, b].tobytes() == oracle.q5_0_block(v[t, g, 32 * b:32 * b + 32])
                assert kb[t, g, b].tobytes() == oracle.q8_0_block(k[t, g, 32 * b:32 * b + 32])


def deq(blocks, fn):
    n, g, nb, _ = blocks.shape
    out = np.zeros((n, g, D))
    for i in range(n):
        for j in range(g):
            out[i, j] = np.concatenate([fn(blocks[i, j, b].tobytes()) for b in range(nb)])
    return out


def test_q5_0_zero_query_is_uniform_mean():
    rng = np.random.default_rng(35)
    n_keys, n_kv, n_qh, n_q = 31, 2, 4, 3
    kb, vb = oracle.quantize_rows(rng.standard_normal((n_keys, n_kv, D)).astype(np.float16),
                                  rng.standard_normal((n_keys, n_kv, D)).astype(np.float16), v_type=Q5)
    vd = deq(vb, oracle.dequant_q5_0)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, np.zeros((n_q, n_qh, D), np.float16), pos0, v_type=Q5)
    for j in range(n_q):
        n_vis = pos0 + j + 1
        for hq in range(n_qh):
            np.testing.assert_allclose(out[j, hq], vd[:n_vis, hq // 2].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[j, hq] - math.log(n_vis)) < 1e-13


def test_q5_0_against_scipy_softmax_random():
    rng = np.random.default_rng(36)
    n_keys, n_kv, n_qh, n_q = 180, 2, 6, 3
    kb, vb = oracle.quantize_rows(rng.standard_normal((n_keys, n_kv, D)).astype(np.float16),
                                  rng.standard_normal((n_keys, n_kv, D)).astype(np.float16), v_type=Q5)
    kd, vd = deq(kb, oracle.dequant_q8_0), deq(vb, oracle.dequant_q5_0)
    q = rng.standard_normal((n_q, n_qh, D)).astype(np.float16)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, q, pos0, v_type=Q5)
    for j in range(n_q):
        for hq in range(n_qh):
            g = hq // 3
            nv = pos0 + j + 1
            s = kd[:nv, g] @ q[j, hq].astype(np.float64) / math.sqrt(D)
            np.testing.assert_allclose(out[j, hq], softmax(s) @ vd[:nv, g], rtol=0, atol=1e-12)
            assert abs(lse[j, hq] - logsumexp(s)) < 1e-12


def test_q5_0_v_error_sits_between_q4_0_and_q8_0():
    """Same inputs and K: only the V quantization differs; against attention
    over the exact fp16 values, Q5_0 V lands between Q8_0 V and Q4_0 V."""
    rng = np.random.default_rng(37)
    n_keys = 150
    k = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    v = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    q = rng.standard_normal((1, 1, D)).astype(np.float16)
    errs = {}
    for vt in (oracle.V_Q4_0, Q5, oracle.V_Q8_0):
        kb, vb = oracle.quantize_rows(k, v, v_type=vt)
        o, l = oracle.attention(kb, vb, q, n_keys - 1, v_type=vt)
        kd = deq(kb, oracle.dequant_q8_0)[:, 0]
        p = softmax(kd @ q[0, 0].astype(np.float64) / math.sqrt(D))
        errs[vt] = np.abs(o[0, 0] - p @ v[:, 0].astype(np.float64)).max()
    assert errs[oracle.V_Q8_0] < errs[Q5] / 4 and errs[Q5] < errs[oracle.V_Q4_0] / 1.5


def test_q5_0_block_size_must_match_the_type():
    kb = np.zeros((2, 1, 4, 34), np.uint8)
    vb = np.zeros((2, 1, 4, 18), np.uint8)
    with pytest.raises(AssertionError):
        oracle.attention(kb, vb, np.zeros((1, 1, D), np.float16), 1, v_type=Q5)
