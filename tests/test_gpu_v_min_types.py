"""The q8_0 / q4_1 and q8_0 / q5_1 K/V pairs (V blocks with a minimum m,
x = d q + m) and q8_0 / f16 (V stored as its fp16 values): the V types whose
decode path feeds the tensor cores p and the V value itself.  Bit-exact pages
against the oracle's blocks, and attention parity on every path (resident,
ring, in-place share, tensor-core verify and prefill widths).  The values carry
1-2 % outliers x8 of both signs, so blocks with a large-magnitude minimum
(where q d and m nearly cancel) occur."""
import numpy as np
import pytest

import oracle
from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, export_page, make_cfg, oracle_blocks, oracle_step, prefill, step, to_dev, torch

pytestmark = pytest.mark.gpu
TYPES = [oracle.V_F16, oracle.V_Q4_1, oracle.V_Q5_1]


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


@pytest.mark.parametrize("vt", TYPES)
def test_pages_are_the_oracle_blocks(kvs, vt):
    w = W.Workload(f"vm{vt}pages", n_layers=1, n_q=1, n_q_heads=8, n_kv_heads=2, ctx=1300,
                   n_resident_pages=2, n_ring_slots=2, seed=71 + vt, outlier_frac=0.02, outlier_scale=8.0)
    cfg = make_cfg(w, type_v=vt)
    h = kvs.kvs_create(cfg, 0)
    try:
        pos = 0
        for n in (1, 37, 256, 300, 5, 700, 1):
            k, v = W.kv_tokens(w, 0, pos, pos + n)
            kvs.kvs_append(h, 0, pos, n, to_dev(k), to_dev(v))
            pos += n
        torch().cuda.synchronize()
        kb, vb = oracle_blocks(w, 0, w.ctx, vt)
        P = w.n_pages
        for p in range(P):
            n = min(256, w.ctx - 256 * p)
            for dev in ((0, 1) if p >= P - w.n_resident_pages else (0,)):
                ek, ev = export_page(h, cfg, 0, p, dev)
                assert np.array_equal(ek[:n], kb[256 * p:256 * p + n])
                assert np.array_equal(ev[:n], vb[256 * p:256 * p + n])
    finally:
        kvs.kvs_destroy(h)


@pytest.mark.parametrize("vt", TYPES)
@pytest.mark.parametrize("ctx,heads,n_q,R,N,pct", [
    (5000, (32, 8), 1, 3, 4, 0),       # ring only, GQA 4
    (5000, (32, 8), 1, 3, 4, 80),      # in-place share + ring
    (4097, (8, 1), 1, 2, 2, 100),      # GQA 8, in place only
    (300, (32, 8), 1, 2, 2, 0),        # short context: few keys per row
    (3000, (40, 8), 4, 2, 4, 0),       # verify width: tensor cores
    (2100, (40, 8), 64, 2, 4, 0),      # three 128-row tiles per kv head
])
def test_attention_parity(kvs, vt, ctx, heads, n_q, R, N, pct):
    w = W.Workload(f"vm{vt}att", n_layers=2, n_q=n_q, n_q_heads=heads[0], n_kv_heads=heads[1], ctx=ctx,
                   n_resident_pages=R, n_ring_slots=N, seed=81 + vt, outlier_frac=0.02, outlier_scale=8.0)
    h = kvs.kvs_create(make_cfg(w, type_v=vt, zero_copy_pct=pct), 0)
    try:
        for layer in range(w.n_layers):
            prefill(h, w, layer, w.pos0)
            out, lse = step(h, w, layer, w.pos0, n_q)
            assert_close(out, lse, *oracle_step(w, layer, w.pos0, n_q, v_type=vt))
    finally:
        kvs.kvs_destroy(h)


@pytest.mark.parametrize("vt", TYPES)
def test_prefill_chunk_width(kvs, vt):
    """256 query tokens (1280 rows per kv head, ten M tiles), sampled rows."""
    w = W.Workload(f"vm{vt}pf", n_layers=1, n_q=256, n_q_heads=40, n_kv_heads=8, ctx=6000,
                   n_resident_pages=4, n_ring_slots=8, seed=91 + vt)
    h = kvs.kvs_create(make_cfg(w, type_v=vt), 0)
    try:
        prefill(h, w, 0, w.pos0)
        out, lse = step(h, w, 0, w.pos0, w.n_q)
        kb, vb = oracle_blocks(w, 0, w.ctx, vt)
        q = W.queries(w, 0, w.pos0)
        for j in (0, 1, 131, 255):
            ro, rl = oracle.attention(kb, vb, q[j:j + 1].copy(), w.pos0 + j, vt)
            assert_close(out[j:j + 1], lse[j:j + 1], ro, rl)
    finally:
        kvs.kvs_destroy(h)


@pytest.mark.parametrize("vt", TYPES)
def test_streaming_equals_all_resident(kvs, vt):
    w = W.Workload(f"vm{vt}eq", n_layers=1, n_q=1, n_q_heads=32, n_kv_heads=8, ctx=3000,
                   n_resident_pages=2, n_ring_slots=4, seed=101 + vt)
    hs = kvs.kvs_create(make_cfg(w, type_v=vt), 0)
    ha = kvs.kvs_create(make_cfg(w, type_v=vt, n_resident_pages=w.n_pages, n_ring_slots=0), 0)
    try:
        outs = []
        for h in (hs, ha):
            prefill(h, w, 0, w.pos0)
            outs.append(step(h, w, 0, w.pos0, 1))
        assert np.allclose(outs[0][0], outs[1][0], rtol=0, atol=2e-5)
        assert np.allclose(outs[0][1], outs[1][1], rtol=0, atol=2e-5)
    finally:
        kvs.kvs_destroy(hs)
        kvs.kvs_destroy(ha)
