"""Parity at the workloads' full sizes, in the configuration bench.py times
(same handle config: layers, resident pages, ring slots, chunking, in-place
share of the streamed pages), on outputs
the oracle can compute one by one: whole layers of the decode and verify
workloads, sampled query tokens of the 256-token prefill chunk."""
import numpy as np
import pytest

import oracle
from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, make_cfg, prefill, step, to_dev, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


def bench_shares(w):
    """The in-place shares bench.py gives this workload: the tuned share of its
    width (decode or the tensor-core path) when pages stream, else none."""
    if w.n_ring_slots == 0:
        return 0, 0
    if w.n_q * (w.n_q_heads // w.n_kv_heads) <= 8:
        return W.ZERO_COPY_PCT, 0
    return 0, W.ZERO_COPY_PCT_WIDE


def _full(kvs, name, layers, sample_q=None):
    t = torch()
    w = W.WORKLOADS[name]
    pct, pct_wide = bench_shares(w)
    h = kvs.kvs_create(make_cfg(w, zero_copy_pct=pct, zero_copy_pct_wide=pct_wide, type_v=w.type_v), 0)
    try:
        for layer in layers:
            prefill(h, w, layer, w.pos0)
            out, lse = step(h, w, layer, w.pos0, w.n_q)
            k, v = W.kv_tokens(w, layer, 0, w.ctx)
            kb, vb = oracle.quantize_rows(k, v, w.type_v)
            q = W.queries(w, layer, w.pos0)
            js = range(w.n_q) if sample_q is None else sample_q
            for j in js:
                ro, rl = oracle.attention(kb, vb, q[j:j + 1].copy(), w.pos0 + j, w.type_v)
                assert_close(out[j:j + 1], lse[j:j + 1], ro, rl)
            st = kvs.kvs_get_stats(h)
            assert st["pages_streamed"] > 0
    finally:
        kvs.kvs_destroy(h)


def test_streamed_decode_32k_full(kvs):
    _full(kvs, "streamed_decode_32k", layers=[0, 15])


def test_streamed_decode_32k_q8v_full(kvs):
    _full(kvs, "streamed_decode_32k_q8v", layers=[3])


def test_streamed_decode_32k_q5v_full(kvs):
    _full(kvs, "streamed_decode_32k_q5v", layers=[9])


def test_long_decode_256k_full(kvs):
    _full(kvs, "long_decode_256k", layers=[7])


def test_verify_128k_full_aux_layer(kvs):
    # the 17th (auxiliary) layer shares the pool with the 16 target layers
    _full(kvs, "verify_128k", layers=[16])


def test_prefill_chunk_64k_sampled(kvs):
    # one query token in each of the ten 128-row M tiles (5 rows per token):
    # token j owns rows 5j..5j+4, so these tokens fall in tiles 0, 1, ..., 9
    _full(kvs, "prefill_chunk_64k", layers=[0],
          sample_q=[0, 26, 52, 77, 103, 128, 154, 180, 205, 231, 255])
