"""Pins of the oracle's page policy: the auto resident-set numbers printed on the
pages (tests/golden/auto_resident.txt), the floor and the ceiling, and the
invariants of the resident/streamed split."""
import pytest

import oracle
from golden_io import read_fixture

PAGE_BYTES_8KV = 8 * 256 * (4 * 34 + 4 * 18)  # one page of 8 kv heads x 128 dims, K Q8_0 + V Q4_0


def test_page_bytes_constant():
    # 32-element blocks: Q8_0 = 2 + 32 bytes, Q4_0 = 2 + 16 bytes; 4 blocks per 128-wide row
    assert PAGE_BYTES_8KV == 425984


def test_auto_resident_matches_printed_numbers():
    _, rows = read_fixture("auto_resident.txt")
    for ctx, tokens in rows:
        pages = oracle.auto_resident_pages(int(ctx), PAGE_BYTES_8KV, 16)
        assert pages * 256 == int(tokens)


def test_auto_resident_floor_and_ceiling():
    # 10 % of 4096 is 1.6 pages; the 2048-token floor gives 8 pages
    assert oracle.auto_resident_pages(4096, PAGE_BYTES_8KV, 1) == 8
    assert oracle.auto_resident_pages(20480, PAGE_BYTES_8KV, 1) == 8
    assert oracle.auto_resident_pages(20481, PAGE_BYTES_8KV, 1) == 9
    # ceiling: 8192 MiB over all layers
    big = 1 << 24  # 16M tokens -> 6554 pages wanted
    cap = (8192 << 20) // (PAGE_BYTES_8KV * 16)
    assert oracle.auto_resident_pages(big, PAGE_BYTES_8KV, 16) == cap
    assert cap < 6554


@pytest.mark.parametrize("n_tokens,R", [(1, 4), (256, 4), (257, 4), (1024, 4), (1025, 4),
                                        (32768, 64), (262144, 103), (5000, 1), (5000, 100)])
def test_page_location_invariants(n_tokens, R):
    P = oracle.pages_for(n_tokens)
    assert P == -(-n_tokens // 256)
    kinds = []
    slots = []
    streamed = []
    for p in range(P):
        kind, idx = oracle.page_location(n_tokens, R, p)
        kinds.append(kind)
        if kind == oracle.PAGE_RESIDENT:
            slots.append(idx)
        else:
            assert kind == oracle.PAGE_STREAMED
            streamed.append(idx)
    # the newest page is always resident
    assert kinds[-1] == oracle.PAGE_RESIDENT
    # resident pages are the min(R, P) most recent, in distinct slots < R
    n_res = min(R, P)
    assert kinds[P - n_res:] == [oracle.PAGE_RESIDENT] * n_res
    assert sorted(slots) == sorted(set(slots)) and all(0 <= s < R for s in slots)
    if P >= R:
        assert sorted(slots) == list(range(R))
    # streamed pages come in ascending order 0..S-1
    assert streamed == list(range(P - n_res))
    # pages beyond the history are absent
    assert oracle.page_location(n_tokens, R, P)[0] == oracle.PAGE_ABSENT
    assert oracle.page_location(n_tokens, R, -1)[0] == oracle.PAGE_ABSENT


def test_slot_is_page_mod_r():
    for p in range(100, 164):
        kind, idx = oracle.page_location(164 * 256, 64, p)
        assert kind == oracle.PAGE_RESIDENT and idx == p % 64
