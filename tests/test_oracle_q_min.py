"""Pins of the oracle's Q4_1 / Q5_1 V blocks (the asymmetric members of the
block family the pages list among the legal cache types; the rule is read as
the block's range split into 15 or 31 steps from its minimum:
d = (max - min)/L, q = min(L, trunc((x - min)/d + 0.5)), x ~ d q + min).

* hand-worked blocks (tests/golden/q4_1_hand.txt, q5_1_hand.txt) with their bytes;
* brute force: every code is the level nearest (x - min)/d, ties upward;
* error bounds, exact constant blocks, and the grid-step relation of the two;
* attention over Q4_1 / Q5_1 V: closed forms and library routines.
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from golden_io import read_fixture

D = 128
TYPES = {
    "q4_1": (oracle.V_Q4_1, 15, 20, oracle.q4_1_block, oracle.dequant_q4_1, "q4_1_hand.txt"),
    "q5_1": (oracle.V_Q5_1, 31, 24, oracle.q5_1_block, oracle.dequant_q5_1, "q5_1_hand.txt"),
}


def h(vals):
    return np.asarray(vals, np.float64).astype(np.float16)


def split(blk: bytes, levels: int):
    """(d bits, m bits, codes), unpacked independently of the oracle."""
    d = int.from_bytes(blk[:2], "little")
    m = int.from_bytes(blk[2:4], "little")
    if levels == 15:
        b = np.frombuffer(blk[4:], np.uint8).astype(int)
        return d, m, np.concatenate([b & 0xF, b >> 4])
    top = int.from_bytes(blk[4:8], "little")
    b = np.frombuffer(blk[8:], np.uint8).astype(int)
    low = np.concatenate([b & 0xF, b >> 4])
    return d, m, low | (np.array([(top >> i) & 1 for i in range(32)]) << 4)


def bits_to_float(bits: int) -> float:
    return float(np.uint16(bits).view(np.float16))


@pytest.mark.parametrize("name", sorted(TYPES))
def test_hand_worked(name):
    vt, levels, nbytes, blockfn, deqfn, fixture = TYPES[name]
    f, _ = read_fixture(fixture)
    # C: division, not a rounded reciprocal; D: the binary32 d, not the stored fp16 d
    for tag in ("A", "B", "C", "D"):
        xs = [float(v) for v in f[f"{tag}_x"]]
        x = h(xs)
        assert np.array_equal(x.astype(np.float64), np.array(xs))  # exact in fp16
        blk = blockfn(x)
        assert len(blk) == nbytes
        d, m, q = split(blk, levels)
        assert d == int(f[f"{tag}_d_bits"][0], 16)
        assert m == int(f[f"{tag}_m_bits"][0], 16)
        if f"{tag}_q" in f:
            assert q.tolist() == [int(v) for v in f[f"{tag}_q"]]
        if f"{tag}_bytes" in f:
            assert list(blk[4:]) == [int(v, 16) for v in f[f"{tag}_bytes"]]
        # the reconstruction is d q + m with the stored fp16 values
        assert np.array_equal(deqfn(blk), bits_to_float(d) * q + bits_to_float(m))
    # A's grid is exact: d and m are short binary fractions
    xa = h([float(v) for v in f["A_x"]])
    qa = np.array([int(v) for v in f["A_q"]])
    da = bits_to_float(int(f["A_d_bits"][0], 16))
    assert np.array_equal(deqfn(blockfn(xa)), da * qa - 1.0)


def _blocks(rng, n):
    for i in range(n):
        kind = i % 4
        if kind == 0:
            x = rng.standard_normal(32)
        elif kind == 1:
            x = rng.uniform(-1, 1, 32) * 10.0 ** rng.integers(-4, 4) + rng.uniform(-3, 3)
        elif kind == 2:  # a short binary grid: many exact ties of the +0.5 rounding
            x = rng.integers(-24, 25, 32) / 8.0
        else:
            x = np.abs(rng.standard_normal(32)) + 2.0  # all positive: min far from 0
        yield h(x)


@pytest.mark.parametrize("name", sorted(TYPES))
def test_brute_force_nearest_level(name):
    """Every code is the step q in 0..L nearest to r = (x - min)/d (binary32),
    ties to the upper step, found by trying all L + 1 steps."""
    vt, levels, nbytes, blockfn, deqfn, fixture = TYPES[name]
    rng = np.random.default_rng(41)
    steps = np.arange(levels + 1)
    for x in _blocks(rng, 400):
        _, _, q = split(blockfn(x), levels)
        xf = x.astype(np.float32)
        lo, hi = xf.min(), xf.max()
        d32 = np.float32(np.float32(hi - lo) / np.float32(levels))
        if d32 == 0:
            assert (q == 0).all()
            continue
        for i in range(32):
            r = float(np.float32(np.float32(xf[i] - lo) / d32))
            dist = np.abs(r - steps)
            want = int(np.flatnonzero(dist == dist.min()).max())
            assert q[i] == want, (i, r, q[i], want)


@pytest.mark.parametrize("name", sorted(TYPES))
def test_error_bound_and_range(name):
    vt, levels, nbytes, blockfn, deqfn, fixture = TYPES[name]
    rng = np.random.default_rng(42)
    for x in _blocks(rng, 1500):
        blk = blockfn(x)
        d_bits, m_bits, q = split(blk, levels)
        xf = x.astype(np.float64)
        lo, hi = xf.min(), xf.max()
        assert m_bits == int(np.float16(lo).view(np.uint16))  # the minimum, exactly
        assert q.min() >= 0 and q.max() <= levels
        deq = deqfn(blk)
        dh = bits_to_float(d_bits)
        assert np.array_equal(deq, dh * q + lo)
        if hi == lo:
            assert (q == 0).all() and np.array_equal(deq, xf)  # constant blocks are exact
            continue
        assert q[int(np.argmin(xf))] == 0
        d32 = float(np.float32(np.float32(hi - lo) / np.float32(levels)))
        tol = d32 * 2 ** -18 + abs(hi) * 2 ** -23 + abs(lo) * 2 ** -23
        assert np.all(np.abs(xf - (d32 * q + lo)) <= d32 / 2 + tol)
        assert np.all(np.abs(xf - deq) <= d32 / 2 + q * abs(dh - d32) + tol)


def test_q5_1_grid_is_twice_as_fine_as_q4_1():
    rng = np.random.default_rng(43)
    se4 = se5 = 0.0
    for _ in range(300):
        x = h(rng.standard_normal(32))
        b4, b5 = oracle.q4_1_block(x), oracle.q5_1_block(x)
        d4 = bits_to_float(int.from_bytes(b4[:2], "little"))
        d5 = bits_to_float(int.from_bytes(b5[:2], "little"))
        assert abs(d5 - d4 * 15 / 31) <= d4 * 2 ** -9
        xf = x.astype(np.float64)
        se4 += float(np.sum((oracle.dequant_q4_1(b4) - xf) ** 2))
        se5 += float(np.sum((oracle.dequant_q5_1(b5) - xf) ** 2))
    assert 0.4 < math.sqrt(se5 / se4) < 0.6


@pytest.mark.parametrize("name", sorted(TYPES))
def test_quantize_rows_matches_blocks(name):
    vt, levels, nbytes, blockfn, deqfn, fixture = TYPES[name]
    rng = np.random.default_rng(44)
    k = rng.standard_normal((4, 2, D)).astype(np.float16)
    v = (rng.standard_normal((4, 2, D)) * 2 + 1).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v, v_type=vt)
    assert kb.shape == (4, 2, 4, 34) and vb.shape == (4, 2, 4, nbytes)
    for t in range(4):
        for g in range(2):
            for b in range(4):
                assert vb[t, g, b].tobytes() == blockfn(v[t, g, 32 * b:32 * b + 32])
                assert kb[t, g, b].tobytes() == oracle.q8_0_block(k[t, g, 32 * b:32 * b + 32])


def deq(blocks, fn):
    n, g, nb, _ = blocks.shape
    out = np.zeros((n, g, D))
    for i in range(n):
        for j in range(g):
            out[i, j] = np.concatenate([fn(blocks[i, j, b].tobytes()) for b in range(nb)])
    return out


@pytest.mark.parametrize("name", sorted(TYPES))
def test_zero_query_is_uniform_mean(name):
    vt, levels, nbytes, blockfn, deqfn, fixture = TYPES[name]
    rng = np.random.default_rng(45)
    n_keys, n_kv, n_qh, n_q = 29, 2, 4, 3
    kb, vb = oracle.quantize_rows(rng.standard_normal((n_keys, n_kv, D)).astype(np.float16),
                                  (rng.standard_normal((n_keys, n_kv, D)) + 0.5).astype(np.float16), v_type=vt)
    vd = deq(vb, deqfn)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, np.zeros((n_q, n_qh, D), np.float16), pos0, v_type=vt)
    for j in range(n_q):
        n_vis = pos0 + j + 1
        for hq in range(n_qh):
            np.testing.assert_allclose(out[j, hq], vd[:n_vis, hq // 2].mean(axis=0), rtol=0, atol=1e-13)
            assert abs(lse[j, hq] - math.log(n_vis)) < 1e-13


@pytest.mark.parametrize("name", sorted(TYPES))
def test_against_scipy_softmax_random(name):
    vt, levels, nbytes, blockfn, deqfn, fixture = TYPES[name]
    rng = np.random.default_rng(46)
    n_keys, n_kv, n_qh, n_q = 170, 2, 6, 3
    kb, vb = oracle.quantize_rows(rng.standard_normal((n_keys, n_kv, D)).astype(np.float16),
                                  rng.standard_normal((n_keys, n_kv, D)).astype(np.float16), v_type=vt)
    kd, vd = deq(kb, oracle.dequant_q8_0), deq(vb, deqfn)
    q = rng.standard_normal((n_q, n_qh, D)).astype(np.float16)
    pos0 = n_keys - n_q
    out, lse = oracle.attention(kb, vb, q, pos0, v_type=vt)
    for j in range(n_q):
        for hq in range(n_qh):
            g = hq // 3
            nv = pos0 + j + 1
            s = kd[:nv, g] @ q[j, hq].astype(np.float64) / math.sqrt(D)
            np.testing.assert_allclose(out[j, hq], softmax(s) @ vd[:nv, g], rtol=0, atol=1e-12)
            assert abs(lse[j, hq] - logsumexp(s)) < 1e-12


def test_constant_v_rows_are_returned_exactly():
    """With every V row the same constant, the min types store it as m with
    d = 0, so the attention output is that constant whatever the weights."""
    rng = np.random.default_rng(47)
    n_keys = 40
    k = rng.standard_normal((n_keys, 1, D)).astype(np.float16)
    v = np.full((n_keys, 1, D), 0.3, np.float16)
    q = rng.standard_normal((2, 1, D)).astype(np.float16)
    for vt in (oracle.V_Q4_1, oracle.V_Q5_1):
        kb, vb = oracle.quantize_rows(k, v, v_type=vt)
        out, _ = oracle.attention(kb, vb, q, n_keys - 2, v_type=vt)
        assert np.allclose(out, float(np.float16(0.3)), rtol=0, atol=1e-15)
