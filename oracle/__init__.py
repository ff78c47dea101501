"""CPU oracle for host-streamed paged quantized KV attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``host_streamed_paged_kvs_b200``) never imports it and shares no code with it.

The arithmetic lives in ``kvs_oracle.c`` (plain C, single thread; quantization
decisions in binary32, attention in binary64).  This module only builds that
file with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvs_oracle.c")
_HDR = os.path.join(_HERE, "kvs_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

PAGE_ABSENT = -1
PAGE_RESIDENT = 1
PAGE_STREAMED = 2


def build(force: bool = False) -> str:
    """Compile kvs_oracle.c into liboracle.so (IEEE arithmetic, no contraction)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def bind(L):
    """Declare the C prototypes on a loaded oracle library and return it."""
    u16p = ctypes.POINTER(ctypes.c_uint16)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    f64p = ctypes.POINTER(ctypes.c_double)
    L.oracle_half_to_double.restype = ctypes.c_double
    L.oracle_half_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_float_to_half.restype = ctypes.c_uint16
    L.oracle_float_to_half.argtypes = [ctypes.c_float]
    L.oracle_q8_0_block.argtypes = [u16p, u8p]
    L.oracle_q4_0_block.argtypes = [u16p, u8p]
    L.oracle_dequant_q8_0.argtypes = [u8p, f64p]
    L.oracle_dequant_q4_0.argtypes = [u8p, f64p]
    L.oracle_q5_0_block.argtypes = [u16p, u8p]
    L.oracle_dequant_q5_0.argtypes = [u8p, f64p]
    L.oracle_q4_1_block.argtypes = [u16p, u8p]
    L.oracle_dequant_q4_1.argtypes = [u8p, f64p]
    L.oracle_q5_1_block.argtypes = [u16p, u8p]
    L.oracle_dequant_q5_1.argtypes = [u8p, f64p]
    L.oracle_quantize_rows.argtypes = [ctypes.c_int, ctypes.c_int, u16p, u16p, u8p, u8p]
    L.oracle_attention.restype = ctypes.c_int
    L.oracle_attention.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p, u8p,
                                   ctypes.c_int, ctypes.c_int, u16p, f64p, f64p]
    L.oracle_quantize_rows_t.restype = ctypes.c_int
    L.oracle_quantize_rows_t.argtypes = [ctypes.c_int, ctypes.c_int, u16p, u16p, u8p, u8p, ctypes.c_int]
    L.oracle_attention_t.restype = ctypes.c_int
    L.oracle_attention_t.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p, u8p,
                                     ctypes.c_int, ctypes.c_int, u16p, f64p, f64p, ctypes.c_int]
    L.oracle_quantize_rows_kv.restype = ctypes.c_int
    L.oracle_quantize_rows_kv.argtypes = [ctypes.c_int, ctypes.c_int, u16p, u16p, u8p, u8p, ctypes.c_int,
                                          ctypes.c_int]
    L.oracle_attention_kv.restype = ctypes.c_int
    L.oracle_attention_kv.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p, u8p,
                                      ctypes.c_int, ctypes.c_int, u16p, f64p, f64p, ctypes.c_int,
                                      ctypes.c_int]
    L.oracle_pages_for.restype = ctypes.c_long
    L.oracle_pages_for.argtypes = [ctypes.c_long, ctypes.c_int]
    L.oracle_auto_resident_pages.restype = ctypes.c_long
    L.oracle_auto_resident_pages.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_long,
                                             ctypes.c_int]
    L.oracle_page_location.restype = ctypes.c_int
    L.oracle_page_location.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_long,
                                       ctypes.c_long, ctypes.POINTER(ctypes.c_int),
                                       ctypes.POINTER(ctypes.c_long)]
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = bind(ctypes.CDLL(_LIB))
    return _lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _as_half_bits(x) -> np.ndarray:
    a = np.asarray(x)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


# --- binary16 conversions -------------------------------------------------

def half_to_double(h) -> np.ndarray:
    h = _as_half_bits(h)
    L = lib()
    return np.array([L.oracle_half_to_double(int(v)) for v in h.ravel()],
                    dtype=np.float64).reshape(h.shape)


def float_to_half(f) -> np.ndarray:
    f = np.asarray(f, dtype=np.float32)
    L = lib()
    return np.array([L.oracle_float_to_half(float(v)) for v in f.ravel()],
                    dtype=np.uint16).reshape(f.shape)


# --- block quantization ---------------------------------------------------

def q8_0_block(x) -> bytes:
    x = _as_half_bits(x).reshape(32)
    out = np.zeros(34, np.uint8)
    lib().oracle_q8_0_block(_ptr(x, ctypes.c_uint16), _ptr(out, ctypes.c_uint8))
    return out.tobytes()


def q4_0_block(x) -> bytes:
    x = _as_half_bits(x).reshape(32)
    out = np.zeros(18, np.uint8)
    lib().oracle_q4_0_block(_ptr(x, ctypes.c_uint16), _ptr(out, ctypes.c_uint8))
    return out.tobytes()


def q5_0_block(x) -> bytes:
    x = _as_half_bits(x).reshape(32)
    out = np.zeros(22, np.uint8)
    lib().oracle_q5_0_block(_ptr(x, ctypes.c_uint16), _ptr(out, ctypes.c_uint8))
    return out.tobytes()


def dequant_q8_0(blk) -> np.ndarray:
    b = np.frombuffer(bytes(blk), np.uint8).copy()
    out = np.zeros(32, np.float64)
    lib().oracle_dequant_q8_0(_ptr(b, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def dequant_q4_0(blk) -> np.ndarray:
    b = np.frombuffer(bytes(blk), np.uint8).copy()
    out = np.zeros(32, np.float64)
    lib().oracle_dequant_q4_0(_ptr(b, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def dequant_q5_0(blk) -> np.ndarray:
    b = np.frombuffer(bytes(blk), np.uint8).copy()
    out = np.zeros(32, np.float64)
    lib().oracle_dequant_q5_0(_ptr(b, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def q4_1_block(x) -> bytes:
    x = _as_half_bits(x).reshape(32)
    out = np.zeros(20, np.uint8)
    lib().oracle_q4_1_block(_ptr(x, ctypes.c_uint16), _ptr(out, ctypes.c_uint8))
    return out.tobytes()


def q5_1_block(x) -> bytes:
    x = _as_half_bits(x).reshape(32)
    out = np.zeros(24, np.uint8)
    lib().oracle_q5_1_block(_ptr(x, ctypes.c_uint16), _ptr(out, ctypes.c_uint8))
    return out.tobytes()


def dequant_q4_1(blk) -> np.ndarray:
    b = np.frombuffer(bytes(blk), np.uint8).copy()
    out = np.zeros(32, np.float64)
    lib().oracle_dequant_q4_1(_ptr(b, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


def dequant_q5_1(blk) -> np.ndarray:
    b = np.frombuffer(bytes(blk), np.uint8).copy()
    out = np.zeros(32, np.float64)
    lib().oracle_dequant_q5_1(_ptr(b, ctypes.c_uint8), _ptr(out, ctypes.c_double))
    return out


V_F16 = 1
V_Q4_0 = 2
V_Q4_1 = 3
V_Q5_0 = 6
V_Q5_1 = 7
V_Q8_0 = 8
_V_BLOCK = {V_F16: 64, V_Q4_0: 18, V_Q4_1: 20, V_Q5_0: 22, V_Q5_1: 24, V_Q8_0: 34}
K_F16 = 1
K_Q8_0 = 8
_K_BLOCK = {K_F16: 64, K_Q8_0: 34}


def quantize_rows(k, v, v_type: int = V_Q4_0, k_type: int = K_Q8_0):
    """k, v: fp16 [..., dim] -> (K blocks [..., dim/32, 34 (Q8_0) or 64 (F16)],
    V blocks [..., dim/32, block bytes of v_type])."""
    k = _as_half_bits(k)
    v = _as_half_bits(v)
    assert k.shape == v.shape
    dim = k.shape[-1]
    rows = int(np.prod(k.shape[:-1]))
    kb = np.zeros(k.shape[:-1] + (dim // 32, _K_BLOCK[k_type]), np.uint8)
    vb = np.zeros(k.shape[:-1] + (dim // 32, _V_BLOCK[v_type]), np.uint8)
    if k_type != K_Q8_0:
        rc = lib().oracle_quantize_rows_kv(rows, dim, _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
                                           _ptr(kb, ctypes.c_uint8), _ptr(vb, ctypes.c_uint8), k_type, v_type)
        assert rc == 0
    elif v_type == V_Q4_0:
        lib().oracle_quantize_rows(rows, dim, _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
                                   _ptr(kb, ctypes.c_uint8), _ptr(vb, ctypes.c_uint8))
    else:
        rc = lib().oracle_quantize_rows_t(rows, dim, _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
                                          _ptr(kb, ctypes.c_uint8), _ptr(vb, ctypes.c_uint8), v_type)
        assert rc == 0
    return kb, vb


# --- attention ------------------------------------------------------------

def attention(k_blocks: np.ndarray, v_blocks: np.ndarray, q, pos0: int, v_type: int = V_Q4_0,
              k_type: int = K_Q8_0):
    """Exact attention over a quantized history.

    k_blocks: uint8 [n_keys, n_kv, dim/32, 34] (Q8_0) or [..., 64] (k_type = K_F16);
    v_blocks: uint8 [n_keys, n_kv, dim/32, 18]
    (Q4_0), or [..., 20 / 22 / 24 / 34 / 64] for v_type = V_Q4_1 / V_Q5_0 / V_Q5_1 / V_Q8_0 / V_F16
    q: fp16 [n_q, n_qh, dim]; query j sits at position pos0+j and sees keys 0..pos0+j.
    Returns (out float64 [n_q, n_qh, dim], lse float64 [n_q, n_qh]).
    """
    q = _as_half_bits(q)
    n_q, n_qh, dim = q.shape
    n_kv = k_blocks.shape[1]
    assert k_blocks.shape[0] >= pos0 + n_q
    kb = np.ascontiguousarray(k_blocks, dtype=np.uint8)
    vb = np.ascontiguousarray(v_blocks, dtype=np.uint8)
    out = np.zeros((n_q, n_qh, dim), np.float64)
    lse = np.zeros((n_q, n_qh), np.float64)
    assert vb.shape[-1] == _V_BLOCK[v_type] and kb.shape[-1] == _K_BLOCK[k_type]
    if k_type != K_Q8_0:
        rc = lib().oracle_attention_kv(n_kv, n_qh, dim, _ptr(kb, ctypes.c_uint8),
                                       _ptr(vb, ctypes.c_uint8), n_q, pos0,
                                       _ptr(q, ctypes.c_uint16), _ptr(out, ctypes.c_double),
                                       _ptr(lse, ctypes.c_double), k_type, v_type)
    elif v_type == V_Q4_0:
        rc = lib().oracle_attention(n_kv, n_qh, dim, _ptr(kb, ctypes.c_uint8),
                                    _ptr(vb, ctypes.c_uint8), n_q, pos0,
                                    _ptr(q, ctypes.c_uint16), _ptr(out, ctypes.c_double),
                                    _ptr(lse, ctypes.c_double))
    else:
        rc = lib().oracle_attention_t(n_kv, n_qh, dim, _ptr(kb, ctypes.c_uint8),
                                      _ptr(vb, ctypes.c_uint8), n_q, pos0,
                                      _ptr(q, ctypes.c_uint16), _ptr(out, ctypes.c_double),
                                      _ptr(lse, ctypes.c_double), v_type)
    if rc != 0:
        raise ValueError(f"oracle_attention rejected its arguments (rc={rc})")
    return out, lse


# --- page policy ----------------------------------------------------------

def pages_for(n_tokens: int, page_tokens: int = 256) -> int:
    return int(lib().oracle_pages_for(n_tokens, page_tokens))


def auto_resident_pages(max_ctx: int, page_bytes: int, n_layers: int,
                        page_tokens: int = 256) -> int:
    return int(lib().oracle_auto_resident_pages(max_ctx, page_tokens, page_bytes, n_layers))


def page_location(n_tokens: int, n_resident: int, page: int, page_tokens: int = 256):
    kind = ctypes.c_int()
    idx = ctypes.c_long()
    lib().oracle_page_location(n_tokens, page_tokens, n_resident, page,
                               ctypes.byref(kind), ctypes.byref(idx))
    return kind.value, idx.value
