"""The phase arena on the GPU: one allocation re-lent between a prefill layout
(wide compute slab, fewer resident pages) and a decode layout (more resident
pages), an auxiliary (draft) layer whose resident pages are pinned at the
arena top, kvs_pin reservations, draft eject and restore.  Across every switch
the pages that become resident are copied from the authoritative host history
(bit-exact against the oracle's blocks) and attention matches the oracle."""
import numpy as np
import pytest

import oracle
from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, export_page, oracle_blocks, oracle_step, prefill, to_dev, torch

pytestmark = pytest.mark.gpu
MIB = 1 << 20


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


def attend(kvs, h, w, layer, pos0, n_q):
    t = torch()
    q = W.queries(w, layer, pos0, n_q)
    out = t.empty((n_q, w.n_q_heads, 128), dtype=t.float32, device="cuda")
    lse = t.empty((n_q, w.n_q_heads), dtype=t.float32, device="cuda")
    kvs.kvs_attend(h, layer, pos0, n_q, to_dev(q), out, lse)
    t.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def check_resident_pages(kvs, h, w, layer, R):
    """Every resident page of the layer, read from the device, is the oracle's blocks."""
    t = torch()
    t.cuda.synchronize()
    kb, vb = oracle_blocks(w, layer, w.ctx)
    cfg = kvs.kvs_get_config(h)
    P = w.n_pages
    for p in range(max(0, P - R), P):
        kind, _ = kvs.kvs_page_location(h, layer, p)
        assert kind == kvs.KVS_PAGE_RESIDENT
        n = min(256, w.ctx - 256 * p)
        ek, ev = export_page(h, cfg, layer, p, 1)
        assert np.array_equal(ek[:n], kb[256 * p:256 * p + n]) and np.array_equal(ev[:n], vb[256 * p:256 * p + n])


def test_phase_switches_pins_and_draft_eject(kvs):
    # 2 target layers + 1 auxiliary (draft) layer, 40/8 heads, a 64-token
    # prefill width (320 rows per kv head: three M tiles), ring of 4 pages
    w = W.Workload("phase", n_layers=3, n_q=64, n_q_heads=40, n_kv_heads=8, ctx=12000,
                   n_resident_pages=0, n_ring_slots=4, seed=181)
    P = w.n_pages
    cfg = kvs.make_config(3, 40, 8, w.ctx, n_ring_slots=4, max_q_tokens=64, arena_bytes=40 * MIB,
                          n_aux_layers=1, aux_resident_pages=6)
    h = kvs.kvs_create(cfg, 0)
    try:
        st0 = kvs.kvs_get_arena(h)
        assert st0["phase_arena"] and st0["phase"] == kvs.KVS_PHASE_PREFILL and st0["width"] == 64
        assert st0["aux_resident_pages"] == 6 and 1 <= st0["n_resident_pages"] < P
        for layer in range(3):
            prefill(h, w, layer, w.ctx)
        # prefill phase: a 64-token chunk on the tensor cores, every tile sampled
        pos0 = w.ctx - 64
        out, lse = attend(kvs, h, w, 0, pos0, 64)
        ro, rl = oracle_step(w, 0, pos0, 64)
        for j in (0, 25, 26, 51, 52, 63):
            assert_close(out[j:j + 1], lse[j:j + 1], ro[j:j + 1], rl[j:j + 1])

        # decode phase at verify width 4: the compute slab shrinks, more pages are resident
        kvs.kvs_set_phase(h, kvs.KVS_PHASE_DECODE, 4)
        st1 = kvs.kvs_get_arena(h)
        assert st1["phase"] == kvs.KVS_PHASE_DECODE and st1["width"] == 4
        assert st1["n_resident_pages"] > st0["n_resident_pages"]
        assert st1["compute_bytes"] < st0["compute_bytes"]
        for layer in (0, 1):
            check_resident_pages(kvs, h, w, layer, st1["n_resident_pages"])
            for n_q in (1, 4):
                p0 = w.ctx - n_q
                assert_close(*attend(kvs, h, w, layer, p0, n_q), *oracle_step(w, layer, p0, n_q))
        check_resident_pages(kvs, h, w, 2, 6)
        assert_close(*attend(kvs, h, w, 2, w.ctx - 1, 1), *oracle_step(w, 2, w.ctx - 1, 1))
        with pytest.raises(kvs.KvsError) as e:
            attend(kvs, h, w, 0, w.ctx - 5, 5)
        assert e.value.code == kvs.KVS_E_WIDTH and "too wide" in kvs.kvs_last_error(h)

        # pins come off the top, below the auxiliary pages and each other
        a = kvs.kvs_pin(h, 1 * MIB)
        b = kvs.kvs_pin(h, 3 * MIB + 5)
        assert a - b == 3 * MIB + 256
        st2 = kvs.kvs_get_arena(h)
        assert st2["pinned_bytes"] == 4 * MIB + 256
        assert st2["n_resident_pages"] <= st1["n_resident_pages"]
        check_resident_pages(kvs, h, w, 0, st2["n_resident_pages"])
        assert_close(*attend(kvs, h, w, 1, w.ctx - 4, 4), *oracle_step(w, 1, w.ctx - 4, 4))

        # draft eject: the pinned region goes back to the target's pages
        kvs.kvs_draft_eject(h)
        st3 = kvs.kvs_get_arena(h)
        assert st3["draft_active"] == 0 and st3["aux_bytes"] == 0 and st3["pinned_bytes"] == 0
        assert st3["n_resident_pages"] > st2["n_resident_pages"]
        with pytest.raises(kvs.KvsError) as e:
            attend(kvs, h, w, 2, w.ctx - 1, 1)
        assert e.value.code == kvs.KVS_E_INVAL
        check_resident_pages(kvs, h, w, 1, st3["n_resident_pages"])
        assert_close(*attend(kvs, h, w, 0, w.ctx - 1, 1), *oracle_step(w, 0, w.ctx - 1, 1))

        # restore: the auxiliary layer's window comes back from the host history
        kvs.kvs_draft_restore(h)
        st4 = kvs.kvs_get_arena(h)
        assert st4["draft_active"] == 1 and st4["aux_resident_pages"] == 6
        check_resident_pages(kvs, h, w, 2, 6)
        assert_close(*attend(kvs, h, w, 2, w.ctx - 4, 4), *oracle_step(w, 2, w.ctx - 4, 4))

        # back to prefill: the wide chunk again
        kvs.kvs_set_phase(h, kvs.KVS_PHASE_PREFILL)
        st5 = kvs.kvs_get_arena(h)
        assert st5["width"] == 64 and st5["n_resident_pages"] == st0["n_resident_pages"]
        out, lse = attend(kvs, h, w, 1, pos0, 64)
        ro, rl = oracle_step(w, 1, pos0, 64)
        for j in (0, 30, 63):
            assert_close(out[j:j + 1], lse[j:j + 1], ro[j:j + 1], rl[j:j + 1])
        kvs.kvs_sync(h, None, 30.0)
    finally:
        kvs.kvs_destroy(h)


def test_no_phase_arena_rejects_phase_calls(kvs):
    h = kvs.kvs_create(kvs.make_config(1, 8, 2, 1000, n_resident_pages=2, n_ring_slots=2), 0)
    try:
        for call in (lambda: kvs.kvs_set_phase(h, kvs.KVS_PHASE_DECODE, 1), lambda: kvs.kvs_pin(h, 4096),
                     lambda: kvs.kvs_draft_eject(h)):
            with pytest.raises(kvs.KvsError) as e:
                call()
            assert e.value.code == kvs.KVS_E_INVAL
        assert kvs.kvs_get_arena(h)["phase_arena"] == 0
    finally:
        kvs.kvs_destroy(h)
