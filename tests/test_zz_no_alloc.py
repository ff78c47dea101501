"""kvs_attend_pages_static: the entry point for callers that cannot allocate
device memory (an engine whose pool owns all device memory, allocations frozen
after start-up, or a loop that must not take cudaMalloc's implicit device
synchronization).  It keeps its split partials in a static device array of the
library instead of allocating.  Its results must match the binary64 oracle and
the handle-based kvs_attend on the same pages, call after call (the array keeps
the previous call's contents, so two calls in a row are checked).

This file is named to be collected last.
"""
import numpy as np
import pytest

from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import LSE_ATOL, O_RTOL_ABS, assert_close, export_page, oracle_step, to_dev, torch

pytestmark = pytest.mark.gpu

PAGE_HEAD = 53248


def internal_page(kb, vb):
    """Canonical blocks of one page -> the library's page layout (per kv head:
    Kq [256][128] | Kd [256][4] fp16 | Vq [256][4][16] | Vd [256][4] fp16)."""
    H = kb.shape[1]
    parts = []
    for h in range(H):
        parts += [kb[:, h, :, 2:].reshape(-1), kb[:, h, :, :2].reshape(-1),
                  vb[:, h, :, 2:].reshape(-1), vb[:, h, :, :2].reshape(-1)]
    page = np.concatenate(parts)
    assert page.size == H * PAGE_HEAD
    return page


def _pages_and_reference(n_tokens, n_q, n_qh, n_kv, seed):
    """The pages written by kvs_append (exported from the resident slots) and
    kvs_attend's out/lse on them for the last n_q positions."""
    t = torch()
    from host_streamed_paged_kvs_b200 import kvs
    w = W.Workload("noalloc", n_layers=1, n_q=n_q, n_q_heads=n_qh, n_kv_heads=n_kv, ctx=n_tokens,
                   n_resident_pages=0, n_ring_slots=0, seed=seed)
    P = -(-n_tokens // 256)
    cfg = kvs.make_config(1, n_qh, n_kv, n_tokens, n_resident_pages=P, n_ring_slots=0, max_q_tokens=n_q)
    h = kvs.kvs_create(cfg, 0)
    try:
        k, v = W.kv_tokens(w, 0, 0, n_tokens)
        kvs.kvs_append(h, 0, 0, n_tokens, to_dev(k), to_dev(v))
        pos0 = n_tokens - n_q
        q = to_dev(W.queries(w, 0, pos0, n_q))
        ref_o = t.empty((n_q, n_qh, 128), dtype=t.float32, device="cuda")
        ref_l = t.empty((n_q, n_qh), dtype=t.float32, device="cuda")
        kvs.kvs_attend(h, 0, pos0, n_q, q, ref_o, ref_l)
        t.cuda.synchronize()
        rcfg = kvs.kvs_get_config(h)
        pages = np.concatenate([internal_page(*export_page(h, rcfg, 0, p, 1)) for p in range(P)])
        return w, P, pos0, q, pages, (ref_o.cpu().numpy(), ref_l.cpu().numpy())
    finally:
        kvs.kvs_destroy(h)


# (n_tokens, n_q, (q heads, kv heads)): 40000 tokens = 157 pages = 314 half-page
# stages, more than the 64 static splits hold, so splits take 5 stages each
CASES = [(3000, 1, (32, 8)), (1500, 4, (16, 2)), (257, 2, (8, 8)), (40000, 1, (40, 8))]


@pytest.mark.parametrize("n_tokens,n_q,heads", CASES)
def test_static_entry_matches_oracle_and_kvs_attend(n_tokens, n_q, heads):
    t = torch()
    from host_streamed_paged_kvs_b200 import kvs
    n_qh, n_kv = heads
    w, P, pos0, q, pages, ref = _pages_and_reference(n_tokens, n_q, n_qh, n_kv, seed=21)
    oref = oracle_step(w, 0, pos0, n_q)
    dpages = t.from_numpy(pages).cuda()
    for _ in range(2):  # two calls in a row share the static scratch
        out = t.full((n_q, n_qh, 128), float("nan"), dtype=t.float32, device="cuda")
        lse = t.full((n_q, n_qh), float("nan"), dtype=t.float32, device="cuda")
        kvs.kvs_attend_pages_static(dpages, P, n_tokens, n_qh, n_kv, pos0, n_q, q, out, lse)
        t.cuda.synchronize()
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        assert_close(o, l, *oref)  # against the binary64 oracle
        ro, rl = ref               # and against kvs_attend, within the same tolerance
        assert np.all(np.abs(o - ro) <= O_RTOL_ABS * (1.0 + np.abs(ro)))
        assert np.all(np.abs(l - rl) <= LSE_ATOL)


def test_static_entry_without_lse_on_a_side_stream():
    """lse = NULL, and a caller stream other than the default one."""
    t = torch()
    from host_streamed_paged_kvs_b200 import kvs
    n_tokens, n_q, n_qh, n_kv = 5000, 2, 16, 4
    w, P, pos0, q, pages, ref = _pages_and_reference(n_tokens, n_q, n_qh, n_kv, seed=22)
    oref = oracle_step(w, 0, pos0, n_q)
    s = t.cuda.Stream()
    with t.cuda.stream(s):
        dpages = t.from_numpy(pages).cuda()
        out = t.full((n_q, n_qh, 128), float("nan"), dtype=t.float32, device="cuda")
        kvs.kvs_attend_pages_static(dpages, P, n_tokens, n_qh, n_kv, pos0, n_q, q, out, None, s)
    s.synchronize()
    o = out.cpu().numpy()
    assert np.all(np.abs(o - oref[0]) <= O_RTOL_ABS * (1.0 + np.abs(oref[0])))
    assert np.all(np.abs(o - ref[0]) <= O_RTOL_ABS * (1.0 + np.abs(ref[0])))


def test_static_entry_rejects_too_many_rows():
    t = torch()
    from host_streamed_paged_kvs_b200 import kvs
    dpages = t.zeros(8 * PAGE_HEAD, dtype=t.uint8, device="cuda")
    q = t.zeros((2, 40, 128), dtype=t.float16, device="cuda")
    out = t.empty((2, 40, 128), dtype=t.float32, device="cuda")
    with pytest.raises(kvs.KvsError) as e:
        kvs.kvs_attend_pages_static(dpages, 1, 256, 40, 8, 254, 2, q, out)
    assert e.value.code == kvs.KVS_E_WIDTH
    assert "64" in kvs.kvs_last_error()
