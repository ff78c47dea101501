"""CPU checks of the C-ABI library: it loads, exports every symbol that
include/kvs.h declares, and its pure host logic (config resolution, auto
sizing, gates, page planning) agrees with the oracle and the pages."""
import ctypes
import os
import re

import pytest

import oracle
from host_streamed_paged_kvs_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvs():
    B.build()
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kvs.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvs_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(kvs):
    names = declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(kvs.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"libkvs.so does not export {n}"
    assert sorted(kvs.EXPORTS) == names


def header_defines(prefix):
    src = open(os.path.join(ROOT, "include", "kvs.h")).read()
    return {m.group(1): int(m.group(2), 0)
            for m in re.finditer(r"#define\s+(" + prefix + r"[A-Z0-9_]+)\s+\(?(-?\w+)\)?", src)}


def test_header_constants_match_binding_and_oracle(kvs):
    """The cache-type, page-kind, flag and error codes of include/kvs.h are the
    binding's, and the V type codes are the oracle's block-type ids."""
    types = header_defines("KVS_TYPE_")
    assert types == {"KVS_TYPE_F16": 1, "KVS_TYPE_Q4_0": 2, "KVS_TYPE_Q4_1": 3, "KVS_TYPE_Q5_0": 6,
                     "KVS_TYPE_Q5_1": 7, "KVS_TYPE_Q8_0": 8}
    for name, val in types.items():
        assert getattr(kvs, name) == val
        assert getattr(oracle, "V_" + name[len("KVS_TYPE_"):]) == val
    for prefix in ("KVS_PAGE_", "KVS_FLAG_"):
        for name, val in header_defines(prefix).items():
            assert getattr(kvs, name) == val, name
    errors = header_defines("KVS_E_")
    assert errors and all(kvs.ERROR_NAMES[v] == k for k, v in errors.items())
    assert kvs.ERROR_NAMES[0] == "KVS_OK"


def test_struct_sizes_match_header(kvs):
    # 14 ints + size_t + 3 ints (padded to 8) ; 8 u64, 6 double, 9 u64, double + 2 u64
    assert ctypes.sizeof(kvs.kvs_config) == 14 * 4 + 8 + 3 * 4 + 4
    assert ctypes.sizeof(kvs.kvs_arena_status) == 6 * 4 + 7 * 8
    assert ctypes.sizeof(kvs.kvs_stats) == (8 + 6 + 9 + 3) * 8


def test_auto_resident_matches_oracle_and_pages(kvs):
    for ctx, L in [(262144, 16), (65536, 16), (4096, 1), (131072, 17), (1 << 24, 16), (20481, 1)]:
        c = kvs.make_config(L, 40, 8, ctx, n_ring_slots=16)
        r, host_bytes = kvs.kvs_resolve_config(c)
        pb = kvs.kvs_page_bytes(r)
        assert pb == 425984
        want = min(oracle.auto_resident_pages(ctx, pb, L), oracle.pages_for(ctx))
        assert r.n_resident_pages == want
        assert host_bytes == L * oracle.pages_for(ctx) * pb
    r, _ = kvs.kvs_resolve_config(kvs.make_config(16, 40, 8, 262144, n_ring_slots=16))
    assert r.n_resident_pages == 103 and r.chunk_pages == 8


def test_plan_page_matches_oracle(kvs):
    for n_tokens, R in [(1, 4), (256, 4), (257, 4), (1025, 4), (32768, 64), (262144, 103), (5000, 1)]:
        c = kvs.make_config(1, 8, 2, max(n_tokens, 1 << 20) if R < 1 << 12 else n_tokens,
                            n_resident_pages=R, n_ring_slots=2)
        r, _ = kvs.kvs_resolve_config(c)
        P = oracle.pages_for(n_tokens)
        for p in list(range(-1, min(P + 1, 300))) + [P - 1, P]:
            assert kvs.kvs_plan_page(r, n_tokens, p) == oracle.page_location(n_tokens, R, p)


@pytest.mark.parametrize("over,code", [
    (dict(type_k=2), -1), (dict(type_v=0), -1), (dict(type_k=8, type_v=4), -1), (dict(type_v=5), -1),
    (dict(type_k=1, type_v=2), -1), (dict(type_k=1, type_v=8), -1),
    (dict(type_v=9), -1),
    (dict(type_k=6, type_v=6), -1), (dict(head_dim=64), -1), (dict(page_tokens=128), -1),
    (dict(n_q_heads=12, n_kv_heads=8), -1), (dict(n_ring_slots=0, n_resident_pages=4), -1),
    (dict(n_ring_slots=6, chunk_pages=4), -1), (dict(arena_bytes=1000), -2),
    (dict(arena_bytes=425984), -2), (dict(max_q_tokens=0), -1), (dict(n_layers=0), -1),
])
def test_gates(kvs, over, code):
    args = dict(n_layers=2, n_q_heads=40, n_kv_heads=8, max_ctx=32768, n_resident_pages=8,
                n_ring_slots=8, max_q_tokens=1)
    args.update(over)
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_resolve_config(kvs.make_config(**args))
    assert e.value.code == code
    assert kvs.kvs_last_error()


def test_q8_0_v_pair_geometry(kvs):
    """The q8_0/q8_0 pair: V codes stored like K's, 69,632 B per page head."""
    c = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8,
                        type_v=kvs.KVS_TYPE_Q8_0)
    r, host = kvs.kvs_resolve_config(c)
    assert kvs.kvs_page_bytes(r) == 8 * 69632
    assert host == 2 * 128 * 8 * 69632
    c4 = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8)
    r4, _ = kvs.kvs_resolve_config(c4)
    assert kvs.kvs_page_bytes(r4) == 8 * 53248
    assert r.arena_bytes - r4.arena_bytes == (2 * 8 + 8) * 8 * (69632 - 53248)


def test_q5_0_v_pair_geometry(kvs):
    """The q8_0/q5_0 pair: Q4_0's V nibbles plus 16 B of fifth bits per token
    and kv head, 57,344 B per page head."""
    c = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8,
                        type_v=kvs.KVS_TYPE_Q5_0)
    r, host = kvs.kvs_resolve_config(c)
    assert r.type_v == kvs.KVS_TYPE_Q5_0
    assert kvs.kvs_page_bytes(r) == 8 * 57344
    assert host == 2 * 128 * 8 * 57344
    c4 = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8)
    r4, _ = kvs.kvs_resolve_config(c4)
    assert r.arena_bytes - r4.arena_bytes == (2 * 8 + 8) * 8 * (57344 - 53248)


@pytest.mark.parametrize("tv,head", [(3, 55296), (7, 59392), (1, 100352)])
def test_min_type_v_pair_geometry(kvs, tv, head):
    """The q8_0/q4_1 and q8_0/q5_1 pairs: Q4_0's (Q5_0's) V fields plus an fp16
    block minimum per token, kv head and block; q8_0/f16: the V values as fp16."""
    c = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8, type_v=tv)
    r, host = kvs.kvs_resolve_config(c)
    assert r.type_v == tv
    assert kvs.kvs_page_bytes(r) == 8 * head
    assert host == 2 * 128 * 8 * head


def test_arena_fit_accepts_exact_size(kvs):
    c = kvs.make_config(2, 40, 8, 32768, n_resident_pages=8, n_ring_slots=8)
    r, _ = kvs.kvs_resolve_config(c)
    c.arena_bytes = r.arena_bytes
    r2, _ = kvs.kvs_resolve_config(c)
    assert r2.arena_bytes == r.arena_bytes
    assert r.arena_bytes >= (2 * 8 + 8) * 425984


@pytest.mark.parametrize("layers,qh,kvh,ctx,ring,mq,budget_mib", [
    (16, 32, 8, 32768, 8, 1, 400), (17, 40, 8, 131072, 16, 4, 2240), (1, 40, 8, 65536, 16, 256, 320),
    (2, 8, 2, 4096, 2, 1, 64), (16, 32, 8, 32768, 8, 1, 100000),
])
def test_arena_budget_sizes_the_resident_set(kvs, layers, qh, kvh, ctx, ring, mq, budget_mib):
    """n_resident_pages = 0 with a fixed arena: the most resident pages that
    fit (one more would not, unless every page already is resident)."""
    budget = budget_mib << 20
    c = kvs.make_config(layers, qh, kvh, ctx, n_ring_slots=ring, max_q_tokens=mq, arena_bytes=budget)
    r, _ = kvs.kvs_resolve_config(c)
    R = r.n_resident_pages
    P = oracle.pages_for(ctx)
    # a phase arena keeps the whole budget as its allocation
    assert 1 <= R <= P and r.arena_bytes == budget and r.flags & kvs.KVS_FLAG_PHASE_ARENA

    def need(n):
        e = kvs.make_config(layers, qh, kvh, ctx, n_resident_pages=n, n_ring_slots=ring, max_q_tokens=mq)
        return kvs.kvs_resolve_config(e)[0].arena_bytes

    assert need(R) <= budget
    if R < P:
        assert need(R + 1) > budget
    # the resident bytes dominate: the grant is the arena minus ring, partials and staging
    assert need(R) >= layers * R * kvs.kvs_page_bytes(r)


@pytest.mark.parametrize("layers,qh,kvh,ctx,ring,mq,budget", [
    (16, 32, 8, 32768, 8, 1, 8 * 425984),             # below ring + one resident page per layer
    (1, 40, 8, 65536, 16, 256, 40 << 20),             # the 256-row split partials alone need more
])
def test_arena_budget_without_room_is_rejected(kvs, layers, qh, kvh, ctx, ring, mq, budget):
    c = kvs.make_config(layers, qh, kvh, ctx, n_ring_slots=ring, max_q_tokens=mq, arena_bytes=budget)
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_resolve_config(c)
    assert e.value.code == kvs.KVS_E_ARENA


def test_create_without_gpu_fails_loudly(kvs):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_create(kvs.make_config(1, 8, 2, 1024), 0)
    assert e.value.code == kvs.KVS_E_CUDA


def test_static_entry_rejects_misaligned_pointers_on_the_host(kvs):
    """kvs_attend_pages_static checks its pointers before any CUDA call, so
    these rejections need no GPU (the addresses are never dereferenced)."""
    base = 1 << 20
    cases = [
        (base + 8, base, base, 0, "pages"),      # pages: TMA and 16-byte copies
        (base, base + 4, base, 0, "8-byte"),     # q: 8-byte words
        (base, base + 2, base, 0, "8-byte"),
        (base, base, base + 2, 0, "4-byte"),     # out: floats
        (base, base, base, base + 1, "4-byte"),  # lse: floats
    ]
    for pages, q, out, lse, what in cases:
        rc = kvs.lib.kvs_attend_pages_static(pages, 4, 1000, 8, 2, 999, 1, q, out, lse or None, None)
        assert rc == kvs.KVS_E_INVAL
        assert what in kvs.kvs_last_error()


def test_zero_copy_share_setter_range(kvs):
    assert kvs.lib.kvs_set_zero_copy_pct(None, 10, -1) == kvs.KVS_E_INVAL
    for over in (dict(zero_copy_pct_wide=101), dict(zero_copy_pct_wide=-1)):
        with pytest.raises(kvs.KvsError):
            kvs.kvs_resolve_config(kvs.make_config(1, 8, 2, 1000, n_ring_slots=2, **over))


def test_f16_f16_pair_geometry_and_gates(kvs):
    """The f16-f16 pair: K and V both stored as fp16 values, 131,072 B per page
    head; F16 K with any other V type is rejected."""
    c = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8,
                        type_k=kvs.KVS_TYPE_F16, type_v=kvs.KVS_TYPE_F16)
    r, host = kvs.kvs_resolve_config(c)
    assert (r.type_k, r.type_v) == (kvs.KVS_TYPE_F16, kvs.KVS_TYPE_F16)
    assert kvs.kvs_page_bytes(r) == 8 * 131072
    assert host == 2 * 128 * 8 * 131072
    for tv in (kvs.KVS_TYPE_Q4_0, kvs.KVS_TYPE_Q8_0, kvs.KVS_TYPE_Q5_1):
        bad = kvs.make_config(2, 32, 8, 32768, n_resident_pages=8, n_ring_slots=8,
                              type_k=kvs.KVS_TYPE_F16, type_v=tv)
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_resolve_config(bad)
        assert e.value.code == kvs.KVS_E_INVAL
        assert "pair" in kvs.kvs_last_error()
