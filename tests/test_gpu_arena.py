"""A handle whose resident set comes from a fixed device arena budget
(n_resident_pages = 0 with arena_bytes set: the decode KV grant of the
arena): parity with the oracle on decode and verify widths, and the arena's
resolved size stays within the budget."""
import pytest

from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, make_cfg, oracle_step, prefill, step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


@pytest.mark.parametrize("budget_mib,n_q,pct", [(12, 1, 80), (12, 4, 0), (20, 1, 0)])
def test_arena_budget_handle_parity(kvs, budget_mib, n_q, pct):
    w = W.Workload("arena", n_layers=2, n_q=n_q, n_q_heads=40, n_kv_heads=8, ctx=9000,
                   n_resident_pages=0, n_ring_slots=4, seed=171)
    cfg = make_cfg(w, max_q_tokens=4, arena_bytes=budget_mib << 20, zero_copy_pct=pct)
    h = kvs.kvs_create(cfg, 0)
    try:
        r = kvs.kvs_get_config(h)
        assert 1 <= r.n_resident_pages < w.n_pages      # the budget, not the context, sets R
        assert r.arena_bytes <= budget_mib << 20
        for layer in range(w.n_layers):
            prefill(h, w, layer, w.pos0)
            out, lse = step(h, w, layer, w.pos0, n_q)
            assert_close(out, lse, *oracle_step(w, layer, w.pos0, n_q))
        assert kvs.kvs_get_stats(h)["pages_streamed"] > 0
    finally:
        kvs.kvs_destroy(h)
