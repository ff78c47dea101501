"""Wide tensor-core calls (more than one 128-row M tile per kv head) send the
last ring chunk as two pieces into the slots of one ring group (8 pages as
5 + 3, 5 as 4 + 1, 3 as 2 + 1; 1 or 2 pages as they are).  Parity with the
oracle for streamed-page counts that give every kind of last chunk, with and
without the in-place share of the streamed pages, over two steps on one handle
(the second reuses the ring groups the first left)."""
import pytest

from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, make_cfg, oracle_step, prefill, step

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("streamed", [1, 2, 3, 5, 8, 9, 13, 17])
@pytest.mark.parametrize("pct_wide", [0, 50])
def test_ring_tail_pieces_match_oracle(streamed, pct_wide):
    from host_streamed_paged_kvs_b200 import kvs
    R = 2
    # 64 query tokens x 5 q heads per kv head = 320 rows: three M tiles
    w = W.Workload("ring_tail", n_layers=1, n_q=64, n_q_heads=40, n_kv_heads=8,
                   ctx=(streamed + R) * W.PAGE_TOKENS, n_resident_pages=R, n_ring_slots=16,
                   seed=40 + streamed)
    h = kvs.kvs_create(make_cfg(w, zero_copy_pct_wide=pct_wide), 0)
    try:
        prefill(h, w, 0, w.pos0)
        for _ in range(2):
            out, lse = step(h, w, 0, w.pos0, w.n_q)
        assert_close(out, lse, *oracle_step(w, 0, w.pos0, w.n_q))
        st = kvs.kvs_get_stats(h)
        assert st["pages_streamed"] == 2 * streamed
    finally:
        kvs.kvs_destroy(h)


# every K/V pair: their raw stages, K^ halves and raw-stage counts differ, and
# with them the shared-memory regions that stage Q and the epilogue's records
@pytest.mark.parametrize("type_k,type_v", [(8, 8), (8, 6), (8, 3), (8, 7), (8, 1), (1, 1)])
@pytest.mark.parametrize("streamed", [8, 13])
def test_ring_tail_every_pair(type_k, type_v, streamed):
    from host_streamed_paged_kvs_b200 import kvs
    R = 2
    w = W.Workload("ring_tail_pair", n_layers=1, n_q=64, n_q_heads=40, n_kv_heads=8,
                   ctx=(streamed + R) * W.PAGE_TOKENS, n_resident_pages=R, n_ring_slots=16,
                   seed=60 + streamed, outlier_frac=0.01, outlier_scale=8.0, type_v=type_v)
    h = kvs.kvs_create(make_cfg(w, type_k=type_k, type_v=type_v), 0)
    try:
        prefill(h, w, 0, w.pos0)
        out, lse = step(h, w, 0, w.pos0, w.n_q)
        assert_close(out, lse, *oracle_step(w, 0, w.pos0, w.n_q, v_type=type_v, k_type=type_k))
    finally:
        kvs.kvs_destroy(h)
