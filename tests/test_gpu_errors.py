"""Error paths of the C ABI on a GPU: every rejection is a status code, none
faults the device, and the handle stays usable afterwards."""
import numpy as np
import pytest

from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import oracle_step, assert_close, prefill, step, to_dev, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


def test_width_order_and_recovery(kvs):
    t = torch()
    w = W.Workload("err", n_layers=1, n_q=1, n_q_heads=8, n_kv_heads=2, ctx=1000,
                   n_resident_pages=2, n_ring_slots=2, seed=5)
    cfg = kvs.make_config(1, 8, 2, 1000, n_resident_pages=2, n_ring_slots=2, max_q_tokens=4)
    h = kvs.kvs_create(cfg, 0)
    try:
        prefill(h, w, 0, 999)
        q = to_dev(W.queries(w, 0, 990, 8))
        out = t.empty((8, 8, 128), dtype=t.float32, device="cuda")
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_attend(h, 0, 990, 8, q, out)       # wider than max_q_tokens
        assert e.value.code == kvs.KVS_E_WIDTH
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_attend(h, 0, 998, 2, q, out)       # query 999 not appended yet
        assert e.value.code == kvs.KVS_E_ORDER
        k, v = W.kv_tokens(w, 0, 0, 1)
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_append(h, 0, 1000, 1, to_dev(k), to_dev(v))  # gap after length 999
        assert e.value.code == kvs.KVS_E_ORDER
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_append(h, 0, 999, 2, to_dev(k), to_dev(v))   # beyond max_ctx
        assert e.value.code == kvs.KVS_E_INVAL
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_attend(h, 3, 0, 1, q, out)           # bad layer
        assert e.value.code == kvs.KVS_E_INVAL
        kh = t.from_numpy(np.zeros((8, 2, 128), np.float16)).pin_memory()
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_append(h, 0, 999, 8, kh, kh)         # host K/V wider than the staging
        assert e.value.code == kvs.KVS_E_WIDTH
        # still usable
        out1, lse1 = step(h, w, 0, 999, 1)
        ref = oracle_step(w, 0, 999, 1)
        assert_close(out1, lse1, *ref)
        kvs.kvs_sync(h, None, 30.0)
    finally:
        kvs.kvs_destroy(h)


def test_create_rejections(kvs):
    bad_pair = kvs.make_config(1, 8, 2, 1000, n_ring_slots=2, type_k=kvs.KVS_TYPE_Q4_0)
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_create(bad_pair, 0)
    assert e.value.code == kvs.KVS_E_INVAL
    tiny_arena = kvs.make_config(1, 8, 2, 1000, n_ring_slots=2, arena_bytes=4096)
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_create(tiny_arena, 0)
    assert e.value.code == kvs.KVS_E_ARENA
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_create(kvs.make_config(1, 8, 2, 1000), 99)
    assert e.value.code == kvs.KVS_E_INVAL


def test_device_bounded_wait_gives_up(kvs):
    """A kernel wait that nothing completes ends after its limit with the
    timeout bit set; the device stays usable."""
    t = torch()
    bits = kvs.kvs_selftest_bounded_wait(0, 0.2)
    assert bits & kvs.KVS_ERR_WAIT_TIMEOUT
    x = t.ones(1024, device="cuda")
    assert float((x * 2).sum().item()) == 2048.0


def test_host_sync_timeout_then_recovers(kvs):
    """kvs_sync's host wait is bounded: a stream still busy returns KVS_E_TIMEOUT;
    waiting longer succeeds."""
    t = torch()
    cfg = kvs.make_config(1, 8, 2, 1024, n_resident_pages=4, n_ring_slots=0)
    h = kvs.kvs_create(cfg, 0)
    try:
        s = t.cuda.Stream()
        with t.cuda.stream(s):
            t.cuda._sleep(1 << 31)  # about a second of GPU clock cycles
        with pytest.raises(kvs.KvsError) as e:
            kvs.kvs_sync(h, s, 0.01)
        assert e.value.code == kvs.KVS_E_TIMEOUT
        kvs.kvs_sync(h, s, 60.0)
    finally:
        kvs.kvs_destroy(h)


def test_misaligned_device_buffers_are_rejected_before_any_launch(kvs):
    """Device Q/out/lse whose addresses the kernels' vector accesses cannot
    take are refused on the host with KVS_E_INVAL; the handle stays usable."""
    t = torch()
    w = W.Workload("align", n_layers=1, n_q=1, n_q_heads=8, n_kv_heads=2, ctx=1000,
                   n_resident_pages=2, n_ring_slots=2, seed=6)
    # 160 q heads: a 7-token batch has 1120 rows, where the merge stores 16-byte words
    cfg = kvs.make_config(1, 8, 2, 1000, n_resident_pages=2, n_ring_slots=2, max_q_tokens=8)
    h = kvs.kvs_create(cfg, 0)
    cfg2 = kvs.make_config(1, 160, 2, 1000, n_resident_pages=2, n_ring_slots=2, max_q_tokens=8)
    h2 = kvs.kvs_create(cfg2, 0)
    try:
        prefill(h, w, 0, 999)
        qbuf = t.zeros(8 * 8 * 128 + 64, dtype=t.float16, device="cuda")
        obuf = t.zeros(8 * 8 * 128 + 64, dtype=t.float32, device="cuda")
        q_ok, out_ok = qbuf.data_ptr(), obuf.data_ptr()

        def rejected(pos0, n_q, q, out, lse=None, handle=h):
            with pytest.raises(kvs.KvsError) as e:
                kvs.kvs_attend(handle, 0, pos0, n_q, q, out, lse)
            assert e.value.code == kvs.KVS_E_INVAL
            return kvs.kvs_last_error(handle)

        assert "8-byte" in rejected(998, 1, q_ok + 4, out_ok)     # decode reads Q in 8-byte words
        assert "16-byte" in rejected(995, 4, q_ok + 8, out_ok)    # 16 rows: tensor-core path
        assert "4-byte" in rejected(998, 1, q_ok, out_ok + 2)
        assert "lse" in rejected(998, 1, q_ok, out_ok, obuf.data_ptr() + 2)
        # the many-row merge writes out in 16-byte words
        w2 = W.Workload("align2", n_layers=1, n_q=7, n_q_heads=160, n_kv_heads=2, ctx=1000,
                        n_resident_pages=2, n_ring_slots=2, seed=6)
        prefill(h2, w2, 0, 999)
        q2 = t.zeros(7 * 160 * 128, dtype=t.float16, device="cuda")
        o2 = t.zeros(7 * 160 * 128 + 16, dtype=t.float32, device="cuda")
        assert "16-byte" in rejected(992, 7, q2, o2.data_ptr() + 4, handle=h2)
        assert kvs.kvs_get_stats(h)["attends"] == 0 and kvs.kvs_get_stats(h2)["attends"] == 0
        # still usable
        out1, lse1 = step(h, w, 0, 999, 1)
        assert_close(out1, lse1, *oracle_step(w, 0, 999, 1))
        kvs.kvs_sync(h, None, 30.0)
    finally:
        kvs.kvs_destroy(h)
        kvs.kvs_destroy(h2)
