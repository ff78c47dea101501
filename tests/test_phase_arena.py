"""The phase arena's host logic (no GPU): one fixed device allocation lent to
a phase (prefill: the widest batch; decode: 1 + n_draft), a pinned region at
its top for the draft (the auxiliary layers' resident pages, then kvs_pin
reservations), and the decode pool that remains ("RaymondHuang210129/
llama.cpp-adaptive-kv-streaming", Summary; "llama.cpp adaptive KV streaming -
spec fork notes", Phase arena: speculative verify batches, New arena and
context API, Dynamic draft eject)."""
import pytest

import oracle


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


MIB = 1 << 20


def cfg(kvs, **over):
    a = dict(n_layers=17, n_q_heads=40, n_kv_heads=8, max_ctx=262144, n_ring_slots=16, max_q_tokens=256,
             arena_bytes=2240 * MIB, n_aux_layers=1)
    a.update(over)
    return kvs.make_config(**a)


def conserved(st):
    parts = ("compute_bytes", "resident_bytes", "ring_bytes", "aux_bytes", "pinned_bytes", "free_bytes")
    return sum(st[p] for p in parts) == st["arena_bytes"]


def test_resolution_keeps_the_budget_and_fits_the_prefill_phase(kvs):
    r, _ = kvs.kvs_resolve_config(cfg(kvs))
    assert r.flags & kvs.KVS_FLAG_PHASE_ARENA
    assert r.arena_bytes == 2240 * MIB
    pb = kvs.kvs_page_bytes(r)
    # the auxiliary layer's window: the 10 % rule (103 pages at 256K)
    assert r.aux_resident_pages == oracle.auto_resident_pages(262144, pb, 1) == 103
    st = kvs.kvs_phase_layout(r, 256)
    assert st["n_resident_pages"] == r.n_resident_pages and st["phase"] == kvs.KVS_PHASE_PREFILL
    assert st["aux_bytes"] == 103 * pb and conserved(st)
    # a resolved config passed back is re-fitted to the same layout
    r2, _ = kvs.kvs_resolve_config(r)
    assert (r2.n_resident_pages, r2.aux_resident_pages, r2.arena_bytes) == \
        (r.n_resident_pages, r.aux_resident_pages, r.arena_bytes)


def test_decode_phase_lends_the_compute_slab_to_resident_pages(kvs):
    r, _ = kvs.kvs_resolve_config(cfg(kvs))
    pre = kvs.kvs_phase_layout(r, 256)
    dec = kvs.kvs_phase_layout(r, 4)   # verify width 1 + 3 drafts
    one = kvs.kvs_phase_layout(r, 1)
    assert pre["compute_bytes"] > dec["compute_bytes"] >= one["compute_bytes"]
    assert pre["n_resident_pages"] < dec["n_resident_pages"] <= one["n_resident_pages"]
    assert dec["phase"] == kvs.KVS_PHASE_DECODE
    for st in (pre, dec, one):
        assert conserved(st)
        # nothing that fits is left unused: one more resident page would not fit
        assert st["free_bytes"] < 16 * kvs.kvs_page_bytes(r) + st["compute_bytes"]


def test_pins_come_off_the_decode_pool_and_eject_returns_them(kvs):
    r, _ = kvs.kvs_resolve_config(cfg(kvs))
    rs = [kvs.kvs_phase_layout(r, 4, m * MIB)["n_resident_pages"] for m in (0, 64, 256, 512)]
    assert rs == sorted(rs, reverse=True) and rs[0] > rs[-1]
    act = kvs.kvs_phase_layout(r, 4, 0, True)
    ej = kvs.kvs_phase_layout(r, 4, 0, False)
    assert ej["aux_bytes"] == 0 and ej["aux_resident_pages"] == 0
    assert ej["n_resident_pages"] > act["n_resident_pages"]
    # the draft-active decode capacity is the same fit (a 4-wide compute slab)
    c4 = cfg(kvs, max_q_tokens=4)
    r4, _ = kvs.kvs_resolve_config(c4)
    assert kvs.kvs_draft_capacity_pages(c4, 64 * MIB) == kvs.kvs_phase_layout(r4, 4, 64 * MIB)["n_resident_pages"]
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_phase_layout(r, 4, 2240 * MIB)
    assert e.value.code == kvs.KVS_E_ARENA


def test_gates(kvs):
    for over in (dict(arena_bytes=0), dict(n_resident_pages=8, arena_bytes=0), dict(n_aux_layers=17),
                 dict(n_aux_layers=-1), dict(aux_resident_pages=-2)):
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_resolve_config(cfg(kvs, **over))
        assert e.value.code == kvs.KVS_E_INVAL
    # a fixed resident count is no phase arena
    r, _ = kvs.kvs_resolve_config(cfg(kvs, n_aux_layers=0, n_resident_pages=8, arena_bytes=0))
    with pytest.raises(kvs.KvsError):
        kvs.kvs_phase_layout(r, 1)
    r, _ = kvs.kvs_resolve_config(cfg(kvs))
    for w in (0, 257):
        with pytest.raises(kvs.KvsError):
            kvs.kvs_phase_layout(r, w)
    # the auxiliary layers' pin alone filling the arena
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_resolve_config(cfg(kvs, arena_bytes=200 * MIB, aux_resident_pages=1024))
    assert e.value.code == kvs.KVS_E_ARENA
