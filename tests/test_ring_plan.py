"""The ring schedule of one attend call (host logic, no GPU), through the C
ABI's kvs_plan_ring, the function kvs_attend itself uses: one copy per chunk
of pages into alternating slot groups, and on the wide tensor-core path the
last chunk as two pieces in one group."""
import pytest

from host_streamed_paged_kvs_b200 import kvs


def _cfg(n_ring_slots=16, chunk_pages=0, heads=(40, 8), max_q=256):
    # all-resident handles (no ring) must hold every page of the context
    c = kvs.make_config(1, heads[0], heads[1], 65536, n_resident_pages=64 if n_ring_slots else 256,
                        n_ring_slots=n_ring_slots, max_q_tokens=max_q, chunk_pages=chunk_pages)
    return kvs.kvs_resolve_config(c)[0]


def _check_invariants(plan, s_ring, cfg):
    chunk, slots = cfg.chunk_pages, cfg.n_ring_slots
    assert sum(p for _, p, _ in plan) == s_ring
    page = 0
    for p0, p, s0 in plan:
        assert p0 == page and 1 <= p <= chunk  # ascending, contiguous pages
        assert 0 <= s0 and s0 + p <= slots     # inside the ring
        # a copy never crosses its group's slots
        assert s0 // chunk == (s0 + p - 1) // chunk
        page += p


def test_prefill_chunk_schedule():
    # 256 query tokens x 5 q heads per kv head: 10 M tiles, the wide path
    cfg = _cfg()
    assert cfg.chunk_pages == 8
    plan = kvs.kvs_plan_ring(cfg, 256, 192)
    _check_invariants(plan, 192, cfg)
    # 23 chunks of 8 pages into alternating groups, then 8 pages as 5 + 3 in
    # the next group
    assert plan[:23] == [(8 * i, 8, 8 * (i % 2)) for i in range(23)]
    assert plan[23:] == [(184, 5, 8), (189, 3, 13)]


def test_decode_schedule_has_no_pieces():
    # one query token: the decode path, whole chunks only (the last one short)
    cfg = _cfg(n_ring_slots=8, heads=(32, 8), max_q=1)
    assert cfg.chunk_pages == 4
    plan = kvs.kvs_plan_ring(cfg, 1, 13)
    _check_invariants(plan, 13, cfg)
    assert plan == [(0, 4, 0), (4, 4, 4), (8, 4, 0), (12, 1, 4)]


def test_single_tile_batches_keep_whole_chunks():
    # verify widths (4 x 5 = 20 rows: one M tile) keep the last chunk whole
    cfg = _cfg()
    plan = kvs.kvs_plan_ring(cfg, 4, 20)
    assert plan == [(0, 8, 0), (8, 8, 8), (16, 4, 0)]


@pytest.mark.parametrize("s_ring,tail", [(1, [(0, 1, 0)]), (2, [(0, 2, 0)]), (3, [(0, 2, 0), (2, 1, 2)]),
                                         (5, [(0, 4, 0), (4, 1, 4)]), (8, [(0, 5, 0), (5, 3, 5)]),
                                         (13, [(8, 4, 8), (12, 1, 12)])])
def test_wide_tail_pieces(s_ring, tail):
    cfg = _cfg()
    plan = kvs.kvs_plan_ring(cfg, 64, s_ring)
    _check_invariants(plan, s_ring, cfg)
    assert plan[-len(tail):] == tail


def test_ring_counter_picks_the_first_group():
    cfg = _cfg()
    even = kvs.kvs_plan_ring(cfg, 256, 40, ring_ctr0=0)
    odd = kvs.kvs_plan_ring(cfg, 256, 40, ring_ctr0=7)
    assert [s for _, _, s in even][:4] == [0, 8, 0, 8]
    assert [s for _, _, s in odd][:4] == [8, 0, 8, 0]
    # the same pages either way, one group apart
    assert [(a, b) for a, b, _ in even] == [(a, b) for a, b, _ in odd]


def test_no_ring_and_bad_arguments():
    cfg = _cfg(n_ring_slots=0)
    assert kvs.kvs_plan_ring(cfg, 256, 0) == []
    cfg = _cfg()
    for n_q, s_ring, ctr in [(0, 8, 0), (1, -1, 0), (1, 8, -1)]:
        with pytest.raises(kvs.KvsError):
            kvs.kvs_plan_ring(cfg, n_q, s_ring, ctr)
