"""Pins of the oracle's Q8_0 / Q4_0 block quantizers.

* hand-worked blocks (tests/golden/q8_0_hand.txt, q4_0_hand.txt);
* closed forms: constant blocks, zero blocks, single non-zero values, sign symmetry;
* the per-block error bounds that the rules imply;
* range invariants (|q| <= 127 with the extreme element at +-127; 0 <= q <= 15 with
  the signed-max element at 0 and its reconstruction exactly -8 d).
"""
import numpy as np
import pytest

import oracle
from golden_io import read_fixture


def h(vals):
    return np.asarray(vals, np.float64).astype(np.float16)


def split_q8(blk: bytes):
    d = int.from_bytes(blk[:2], "little")
    q = np.frombuffer(blk[2:], np.int8).astype(int)
    return d, q


def split_q4(blk: bytes):
    d = int.from_bytes(blk[:2], "little")
    b = np.frombuffer(blk[2:], np.uint8).astype(int)
    q = np.concatenate([b & 0xF, b >> 4])
    return d, q


def test_q8_0_hand_worked():
    f, _ = read_fixture("q8_0_hand.txt")
    x = h([float(v) for v in f["x"]])
    assert np.array_equal(x.astype(np.float64), np.array([float(v) for v in f["x"]]))
    d, q = split_q8(oracle.q8_0_block(x))
    assert d == int(f["d_bits"][0], 16)
    assert q.tolist() == [int(v) for v in f["q"]]
    # C: the code of a correctly rounded x / d (a rounded 1/d would flip it);
    # D: the code with the binary32 d as divisor (the stored fp16 d would flip it)
    for tag in ("C", "D"):
        xs = [float(v) for v in f[f"{tag}_x"]]
        x = h(xs)
        assert np.array_equal(x.astype(np.float64), np.array(xs))
        d, q = split_q8(oracle.q8_0_block(x))
        assert d == int(f[f"{tag}_d_bits"][0], 16), tag
        assert q.tolist() == [int(v) for v in f[f"{tag}_q"]], tag


def test_q4_0_hand_worked():
    f, _ = read_fixture("q4_0_hand.txt")
    # C: division, not a rounded reciprocal; D: the binary32 d, not the stored fp16 d
    for tag in ("A", "B", "C", "D"):
        xs = [float(v) for v in f[f"{tag}_x"]]
        x = h(xs)
        assert np.array_equal(x.astype(np.float64), np.array(xs))  # exact in fp16
        blk = oracle.q4_0_block(x)
        d, q = split_q4(blk)
        assert d == int(f[f"{tag}_d_bits"][0], 16)
        assert q.tolist() == [int(v) for v in f[f"{tag}_q"]]
    blk = oracle.q4_0_block(h([float(v) for v in f["A_x"]]))
    assert list(blk[2:]) == [int(v, 16) for v in f["A_bytes"]]


@pytest.mark.parametrize("c", [1.0, 0.5, 3.0, 1e-3, 60000.0, 2.0 ** -24])
def test_constant_block(c):
    x = h([c] * 32)
    d, q = split_q8(oracle.q8_0_block(x))
    assert (q == 127).all()
    cf = float(x[0])
    # d = fp16(c/127) in binary32
    assert d == int(np.float16(np.float32(cf) / np.float32(127.0)).view(np.uint16))
    d4, q4 = split_q4(oracle.q4_0_block(x))
    assert (q4 == 0).all()
    # d = c / -8 is exact whenever it is a normal fp16 value
    if cf >= 2.0 ** -11:
        assert d4 == int(np.float16(-cf / 8).view(np.uint16))
    d4n, q4n = split_q4(oracle.q4_0_block(-x))
    assert (q4n == 0).all()


def test_zero_block():
    x = h([0.0] * 32)
    assert oracle.q8_0_block(x) == bytes(34)
    d, q = split_q4(oracle.q4_0_block(x))
    # m = +0, so d = +0 / -8 = -0 (fp16 bits 0x8000) and every code is 8
    assert d == 0x8000 and (q == 8).all()
    assert (oracle.dequant_q4_0(oracle.q4_0_block(x)) == 0).all()


@pytest.mark.parametrize("i", [0, 7, 16, 31])
@pytest.mark.parametrize("val", [1.0, -2.5, 0.001])
def test_single_nonzero(i, val):
    x = np.zeros(32, np.float16)
    x[i] = val
    d, q = split_q8(oracle.q8_0_block(x))
    expect = np.zeros(32, int)
    expect[i] = 127 if val > 0 else -127
    assert q.tolist() == expect.tolist()
    d4, q4 = split_q4(oracle.q4_0_block(x))
    e4 = np.full(32, 8)
    e4[i] = 0
    assert q4.tolist() == e4.tolist()
    # the signed-max element reconstructs to -8 d exactly
    deq = oracle.dequant_q4_0(oracle.q4_0_block(x))
    dh = np.uint16(d4).view(np.float16).astype(np.float64)
    assert deq[i] == -8 * dh


def test_q8_0_sign_symmetry():
    rng = np.random.default_rng(5)
    for _ in range(200):
        x = rng.standard_normal(32).astype(np.float16)
        d1, q1 = split_q8(oracle.q8_0_block(x))
        d2, q2 = split_q8(oracle.q8_0_block(-x))
        assert d1 == d2 and (q1 == -q2).all()


def _blocks(rng, n):
    for i in range(n):
        scale = float(np.exp2(rng.uniform(-12, 10)))
        x = rng.standard_normal(32) * scale
        if i % 3 == 0:
            x = np.where(rng.random(32) < 0.1, x * 8, x)
        x = np.clip(x, -60000, 60000).astype(np.float16)
        yield x


def test_q8_0_error_bound_and_range():
    rng = np.random.default_rng(6)
    for x in _blocks(rng, 1500):
        blk = oracle.q8_0_block(x)
        d_bits, q = split_q8(blk)
        xf = x.astype(np.float64)
        amax = np.abs(xf).max()
        d32 = float(np.float32(np.float32(amax) / np.float32(127)))
        dh = float(np.uint16(d_bits).view(np.float16))
        assert np.abs(q).max() <= 127
        assert abs(q[np.argmax(np.abs(xf))]) == 127
        deq = oracle.dequant_q8_0(blk)
        assert np.array_equal(deq, dh * q)
        # |x - d q| <= d32/2 (+ rounding slack of the binary32 quotient) + 127 |d - d32|
        bound = d32 / 2 * (1 + 2 ** -20) + 127 * abs(dh - d32)
        assert np.all(np.abs(xf - deq) <= bound + 1e-300)


def test_q4_0_error_bound_and_range():
    rng = np.random.default_rng(7)
    for x in _blocks(rng, 1500):
        blk = oracle.q4_0_block(x)
        d_bits, q = split_q4(blk)
        xf = x.astype(np.float64)
        i_max = int(np.argmax(np.abs(xf)))  # first index of the largest magnitude
        m = xf[i_max]
        d32 = float(np.float32(np.float32(m) / np.float32(-8)))
        dh = float(np.uint16(d_bits).view(np.float16))
        assert q.min() >= 0 and q.max() <= 15
        assert q[i_max] == 0
        deq = oracle.dequant_q4_0(blk)
        assert np.array_equal(deq, dh * (q - 8))
        ratio = xf / d32
        clamped = ratio > 7.5
        err32 = np.abs(xf - (q - 8) * d32)
        tol = abs(d32) * 2 ** -20
        assert np.all(err32[~clamped] <= abs(d32) / 2 + tol)
        assert np.all(err32[clamped] <= abs(d32) + tol)
        extra = np.abs(q - 8) * abs(dh - d32)
        assert np.all(np.abs(xf - deq) <= err32 + extra + tol)
        assert deq[i_max] == -8 * dh


def test_quantize_rows_matches_blocks():
    rng = np.random.default_rng(8)
    k = rng.standard_normal((3, 2, 128)).astype(np.float16)
    v = rng.standard_normal((3, 2, 128)).astype(np.float16)
    kb, vb = oracle.quantize_rows(k, v)
    assert kb.shape == (3, 2, 4, 34) and vb.shape == (3, 2, 4, 18)
    for t in range(3):
        for g in range(2):
            for b in range(4):
                assert kb[t, g, b].tobytes() == oracle.q8_0_block(k[t, g, b * 32:(b + 1) * 32])
                assert vb[t, g, b].tobytes() == oracle.q4_0_block(v[t, g, b * 32:(b + 1) * 32])
