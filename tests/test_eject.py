"""Draft eject controller ("llama.cpp adaptive KV streaming - spec fork notes",
Dynamic draft eject and Results): pure host logic behind the C ABI.

The rules tested, as the page states them:
- one eject threshold in 256-token pages of the target's decode working set;
  0 ejects at streaming onset, i.e. when the working set outgrows the
  draft-active decode capacity;
- re-enable once the working set fits the given number of pages below the
  threshold (default 8);
- a transition needs that many consecutive decode batches (default 4);
- the draft is never ejected while the working set fits;
- a large keep threshold keeps the draft throughout.
"""
import pytest

from host_streamed_paged_kvs_b200 import kvs as K


def run(params, state, trace):
    """Feed a working-set trace; return the list of (batch index, active after)."""
    events = []
    for i, w in enumerate(trace):
        if K.kvs_eject_step(params, state, w):
            events.append((i, state.draft_active))
    return events


def test_defaults_and_threshold_choice():
    p, s = K.kvs_eject_init(capacity_pages=180)
    assert (p.reenable_pages, p.stable_decodes, p.keep_pages) == (8, 4, 0)
    assert s.draft_active == 1 and s.streak == 0
    # keep_pages = 0: the threshold is the capacity (streaming onset)
    assert run(p, s, [180] * 20) == []
    assert run(p, s, [181] * 4) == [(3, 0)]
    # a positive keep_pages overrides the capacity
    p2, s2 = K.kvs_eject_init(keep_pages=300, capacity_pages=180)
    assert run(p2, s2, [250] * 50) == []
    assert run(p2, s2, [301] * 4) == [(3, 0)]


def test_never_ejected_while_the_working_set_fits():
    p, s = K.kvs_eject_init(capacity_pages=200)
    assert run(p, s, list(range(0, 201)) * 3) == []
    assert s.draft_active == 1


def test_stability_count_and_reset():
    p, s = K.kvs_eject_init(keep_pages=100, stable_decodes=3)
    # two batches above, one back below: the streak restarts
    assert run(p, s, [101, 101, 100, 101, 101]) == []
    assert s.streak == 2
    assert run(p, s, [150]) == [(0, 0)]
    assert s.streak == 0


def test_hysteresis_band_keeps_the_draft_ejected():
    p, s = K.kvs_eject_init(keep_pages=100)  # re-enable at <= 92, 4 batches
    run(p, s, [120] * 4)
    assert s.draft_active == 0
    # inside (92, 100]: stays ejected however long
    assert run(p, s, [100, 99, 95, 93] * 10) == []
    # at 92: re-enabled on the 4th consecutive batch
    assert run(p, s, [92, 92, 92, 92]) == [(3, 1)]
    # and ejected again only above 100
    assert run(p, s, [100] * 10) == []


def test_growing_context_trace():
    """A decode that appends one token per batch from 47K tokens on, with the
    draft-active capacity at 190 pages: the working set (pages of the context)
    passes 190 at token 190*256+1, and the draft is ejected four batches later."""
    p, s = K.kvs_eject_init(capacity_pages=190)
    start = 47 * 1024
    ctx = list(range(start, start + 2000))
    pages = [(c + 255) // 256 for c in ctx]
    ev = run(p, s, pages)
    first_over = next(i for i, w in enumerate(pages) if w > 190)
    assert ev == [(first_over + 3, 0)]


def test_keep_arm_never_ejects():
    p, s = K.kvs_eject_init(keep_pages=1 << 30, capacity_pages=180)
    assert run(p, s, [640] * 100) == []


@pytest.mark.parametrize("kw", [dict(), dict(keep_pages=-1, capacity_pages=5),
                                dict(capacity_pages=5, stable_decodes=-2)])
def test_bad_parameters(kw):
    with pytest.raises(K.KvsError) as e:
        K.kvs_eject_init(**kw)
    assert e.value.code == K.KVS_E_INVAL


def test_negative_working_set_is_rejected():
    p, s = K.kvs_eject_init(capacity_pages=10)
    with pytest.raises(K.KvsError):
        K.kvs_eject_step(p, s, -1)


@pytest.mark.parametrize("pinned_mib", [0, 64, 256, 1024])
def test_draft_capacity_is_the_resident_fit_of_the_remaining_arena(pinned_mib):
    arena = 2240 << 20
    c = K.make_config(17, 40, 8, 262144, n_ring_slots=16, max_q_tokens=4, arena_bytes=arena)
    cap = K.kvs_draft_capacity_pages(c, pinned_mib << 20)
    r, _ = K.kvs_resolve_config(K.make_config(17, 40, 8, 262144, n_ring_slots=16, max_q_tokens=4,
                                              arena_bytes=arena - (pinned_mib << 20)))
    assert cap == r.n_resident_pages


def test_draft_capacity_shrinks_with_the_pin_and_needs_an_arena():
    c = K.make_config(17, 40, 8, 262144, n_ring_slots=16, max_q_tokens=4, arena_bytes=2240 << 20)
    caps = [K.kvs_draft_capacity_pages(c, m << 20) for m in (0, 100, 200, 400)]
    assert caps == sorted(caps, reverse=True) and caps[0] > caps[-1]
    with pytest.raises(K.KvsError) as e:
        K.kvs_draft_capacity_pages(c, 2240 << 20)
    assert e.value.code == K.KVS_E_ARENA
    with pytest.raises(K.KvsError) as e:
        K.kvs_draft_capacity_pages(K.make_config(17, 40, 8, 262144, n_ring_slots=16), 0)
    assert e.value.code == K.KVS_E_INVAL
