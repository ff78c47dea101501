"""Zero-copy decode (zero_copy_pct): the decode kernel reads a share of the
streamed pages in place from the mapped pinned history while the ring brings
the rest.  Parity against the oracle, agreement with the ring-only path on the
same inputs, and the ring still serving the calls too wide for the CUDA-core
kernel."""
import numpy as np
import pytest

from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, make_cfg, oracle_step, prefill, step, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


@pytest.mark.parametrize("ctx,heads,n_q,R,N,pct", [
    (5000, (32, 8), 1, 3, 4, 100),     # ragged last page, GQA 4, no ring copies
    (5000, (32, 8), 1, 3, 4, 60),      # 10 of 17 streamed pages in place, 7 through the ring
    (4097, (8, 1), 1, 2, 2, 100),      # GQA 8: 8 rows per kv head
    (4097, (8, 1), 1, 2, 2, 33),
    (2600, (16, 8), 2, 1, 2, 50),      # two query tokens x GQA 2
    (700, (8, 2), 1, 1, 2, 100),       # three pages, two streamed
    (700, (8, 2), 1, 1, 2, 10),        # rounds to zero pages in place
])
def test_zero_copy_matches_oracle_and_ring(kvs, ctx, heads, n_q, R, N, pct):
    w = W.Workload("zc", n_layers=2, n_q=n_q, n_q_heads=heads[0], n_kv_heads=heads[1], ctx=ctx,
                   n_resident_pages=R, n_ring_slots=N, seed=41)
    hz = kvs.kvs_create(make_cfg(w, zero_copy_pct=pct), 0)
    hr = kvs.kvs_create(make_cfg(w), 0)
    try:
        for layer in range(w.n_layers):
            for h in (hz, hr):
                prefill(h, w, layer, w.pos0)
            oz, lz = step(hz, w, layer, w.pos0, n_q)
            orr, lr = step(hr, w, layer, w.pos0, n_q)
            assert_close(oz, lz, *oracle_step(w, layer, w.pos0, n_q))
            # same arithmetic, other split layout: fp32 rounding apart only
            assert np.allclose(oz, orr, rtol=0, atol=2e-5) and np.allclose(lz, lr, rtol=0, atol=2e-5)
        st = kvs.kvs_get_stats(hz)
        S = w.n_pages - R
        zc = min(S, (S * pct + 50) // 100)
        assert st["pages_streamed"] == w.n_layers * S
        assert (st["h2d_copies"] == 0) == (zc == S)
    finally:
        kvs.kvs_destroy(hz)
        kvs.kvs_destroy(hr)


def test_wide_calls_keep_the_ring(kvs):
    """A verify batch (4 tokens x GQA 5 = 20 rows) goes to the tensor-core
    kernel through the ring even with zero-copy set."""
    w = W.Workload("zcw", n_layers=1, n_q=4, n_q_heads=40, n_kv_heads=8, ctx=3000,
                   n_resident_pages=2, n_ring_slots=4, seed=43)
    h = kvs.kvs_create(make_cfg(w, zero_copy_pct=100), 0)
    p0 = w.ctx - 10
    try:
        prefill(h, w, 0, p0)
        out, lse = step(h, w, 0, p0, 4)
        assert_close(out, lse, *oracle_step(w, 0, p0, 4))
        assert kvs.kvs_get_stats(h)["h2d_copies"] > 0
        # and a single-token decode on the same handle reads in place
        kvs.kvs_reset_stats(h)
        out1, lse1 = step(h, w, 0, p0 + 4, 1)
        assert_close(out1, lse1, *oracle_step(w, 0, p0 + 4, 1))
        assert kvs.kvs_get_stats(h)["h2d_copies"] == 0
    finally:
        kvs.kvs_destroy(h)


@pytest.mark.parametrize("n_q,ctx,R,N,pct", [
    (4, 5000, 3, 4, 100),     # verify width: one M tile per kv head, every streamed page in place
    (4, 5000, 3, 4, 60),      # in place and through the ring in one call
    (64, 3000, 2, 4, 100),    # three M tiles: two tile pairs per kv head
    (256, 6000, 4, 8, 80),    # a prefill chunk: ten M tiles
])
def test_wide_zero_copy_matches_oracle_and_ring(kvs, n_q, ctx, R, N, pct):
    """Calls on the tensor-core path read the wide share of the streamed pages
    in place (16-byte asynchronous copies from the mapped history): parity with
    the oracle (sampled query tokens in every tile for wide batches) and with the
    ring-only path on the same inputs."""
    w = W.Workload("zcwide", n_layers=1, n_q=n_q, n_q_heads=40, n_kv_heads=8, ctx=ctx,
                   n_resident_pages=R, n_ring_slots=N, seed=44)
    hz = kvs.kvs_create(make_cfg(w, zero_copy_pct_wide=pct), 0)
    hr = kvs.kvs_create(make_cfg(w), 0)
    try:
        for h in (hz, hr):
            prefill(h, w, 0, w.pos0)
        oz, lz = step(hz, w, 0, w.pos0, n_q)
        orr, lr = step(hr, w, 0, w.pos0, n_q)
        ro, rl = oracle_step(w, 0, w.pos0, n_q)
        rows = range(n_q) if n_q <= 4 else sorted({0, n_q // 3, n_q // 2, n_q - 1} | set(range(0, n_q, 26)))
        for j in rows:
            assert_close(oz[j:j + 1], lz[j:j + 1], ro[j:j + 1], rl[j:j + 1])
        # same arithmetic, other split layout: each split keeps its own
        # reference max, so P rounds to fp16 at other scales (out within
        # 2^-11 of the weights' share); l is summed in fp32 before rounding
        assert np.allclose(oz, orr, rtol=0, atol=1e-4) and np.allclose(lz, lr, rtol=0, atol=2e-5)
        st = kvs.kvs_get_stats(hz)
        S = w.n_pages - R
        zc = min(S, (S * pct + 50) // 100)
        assert st["pages_streamed"] == S
        assert (st["h2d_copies"] == 0) == (zc == S)
    finally:
        kvs.kvs_destroy(hz)
        kvs.kvs_destroy(hr)


def test_zero_copy_full_size_32k_layer(kvs):
    """The 32K decode workload's layer 0 in the bench configuration, a share of
    the streamed pages in place."""
    w = W.WORKLOADS["streamed_decode_32k"]
    h = kvs.kvs_create(make_cfg(w, zero_copy_pct=W.ZERO_COPY_PCT), 0)
    try:
        prefill(h, w, 0, w.pos0)
        out, lse = step(h, w, 0, w.pos0, 1)
        assert_close(out, lse, *oracle_step(w, 0, w.pos0, 1))
        assert kvs.kvs_get_stats(h)["pages_streamed"] == w.n_pages - w.n_resident_pages
    finally:
        torch().cuda.synchronize()
        kvs.kvs_destroy(h)
