"""The f16-f16 K/V pair (K and V stored as their fp16 values; the pair the
flash-attention build always compiles): bit-exact pages against the oracle's
blocks, and attention parity on every path (resident, ring, in-place share,
tensor-core verify and prefill widths) against the binary64 oracle over the
exact values."""
import numpy as np
import pytest

import oracle
from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, export_page, make_cfg, oracle_blocks, oracle_step, prefill, step, to_dev, torch

pytestmark = pytest.mark.gpu
KF, VF = oracle.K_F16, oracle.V_F16


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


def test_pages_are_the_oracle_blocks(kvs):
    w = W.Workload("f16pages", n_layers=1, n_q=1, n_q_heads=8, n_kv_heads=2, ctx=1300,
                   n_resident_pages=2, n_ring_slots=2, seed=131, outlier_frac=0.02, outlier_scale=8.0)
    cfg = make_cfg(w, type_v=VF, type_k=KF)
    h = kvs.kvs_create(cfg, 0)
    try:
        pos = 0
        for n in (1, 37, 256, 300, 5, 700, 1):
            k, v = W.kv_tokens(w, 0, pos, pos + n)
            kvs.kvs_append(h, 0, pos, n, to_dev(k), to_dev(v))
            pos += n
        torch().cuda.synchronize()
        kb, vb = oracle_blocks(w, 0, w.ctx, VF, KF)
        P = w.n_pages
        rcfg = kvs.kvs_get_config(h)
        for p in range(P):
            n = min(256, w.ctx - 256 * p)
            for dev in ((0, 1) if p >= P - w.n_resident_pages else (0,)):
                ek, ev = export_page(h, rcfg, 0, p, dev)
                assert np.array_equal(ek[:n], kb[256 * p:256 * p + n])
                assert np.array_equal(ev[:n], vb[256 * p:256 * p + n])
    finally:
        kvs.kvs_destroy(h)


@pytest.mark.parametrize("ctx,heads,n_q,R,N,pct", [
    (5000, (32, 8), 1, 3, 4, 0),       # ring only, GQA 4
    (5000, (32, 8), 1, 3, 4, 80),      # in-place share + ring
    (4097, (8, 1), 1, 2, 2, 100),      # GQA 8, in place only
    (300, (32, 8), 1, 2, 2, 0),        # short context: few keys per row
    (3000, (40, 8), 4, 2, 4, 0),       # verify width: tensor cores
    (2100, (40, 8), 64, 2, 4, 0),      # three 128-row tiles per kv head
])
def test_attention_parity(kvs, ctx, heads, n_q, R, N, pct):
    w = W.Workload("f16att", n_layers=2, n_q=n_q, n_q_heads=heads[0], n_kv_heads=heads[1], ctx=ctx,
                   n_resident_pages=R, n_ring_slots=N, seed=141, outlier_frac=0.02, outlier_scale=8.0)
    h = kvs.kvs_create(make_cfg(w, type_v=VF, type_k=KF, zero_copy_pct=pct), 0)
    try:
        for layer in range(w.n_layers):
            prefill(h, w, layer, w.pos0)
            out, lse = step(h, w, layer, w.pos0, n_q)
            assert_close(out, lse, *oracle_step(w, layer, w.pos0, n_q, v_type=VF, k_type=KF))
    finally:
        kvs.kvs_destroy(h)


def test_prefill_chunk_width_every_tile(kvs):
    """256 query tokens (1280 rows per kv head, ten M tiles in five tile
    pairs): one sampled query token in every tile."""
    w = W.Workload("f16pf", n_layers=1, n_q=256, n_q_heads=40, n_kv_heads=8, ctx=6000,
                   n_resident_pages=4, n_ring_slots=8, seed=151)
    h = kvs.kvs_create(make_cfg(w, type_v=VF, type_k=KF), 0)
    try:
        prefill(h, w, 0, w.pos0)
        out, lse = step(h, w, 0, w.pos0, w.n_q)
        kb, vb = oracle_blocks(w, 0, w.ctx, VF, KF)
        q = W.queries(w, 0, w.pos0)
        for j in (0, 26, 52, 77, 103, 128, 154, 180, 205, 231, 255):
            ro, rl = oracle.attention(kb, vb, q[j:j + 1].copy(), w.pos0 + j, VF, KF)
            assert_close(out[j:j + 1], lse[j:j + 1], ro, rl)
    finally:
        kvs.kvs_destroy(h)


def test_streaming_equals_all_resident(kvs):
    w = W.Workload("f16eq", n_layers=1, n_q=1, n_q_heads=32, n_kv_heads=8, ctx=3000,
                   n_resident_pages=2, n_ring_slots=4, seed=161)
    hs = kvs.kvs_create(make_cfg(w, type_v=VF, type_k=KF), 0)
    ha = kvs.kvs_create(make_cfg(w, type_v=VF, type_k=KF, n_resident_pages=w.n_pages, n_ring_slots=0), 0)
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
