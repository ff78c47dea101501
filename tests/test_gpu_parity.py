"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Blocks and page indexing must match bit for bit; attention output within
|out - ref| <= 1e-3 (1 + |ref|) and lse within 1e-4 of the binary64 oracle.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import (assert_close, export_page, make_cfg, oracle_blocks, oracle_step, prefill,
                         step, to_dev, torch)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvs():
    t = torch()
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from host_streamed_paged_kvs_b200 import kvs as K
    return K


def small(name, **kw):
    base = dict(name=name, n_layers=2, n_q=1, n_q_heads=8, n_kv_heads=2, ctx=3000,
                n_resident_pages=3, n_ring_slots=4, seed=11)
    base.update(kw)
    return W.Workload(**base)


# ---------------------------------------------------------------------------
# quantize-on-append: bit-exact blocks, host history and resident slots
# ---------------------------------------------------------------------------
def _check_pages(kvs, h, w, layer, n_tokens):
    cfg = kvs.kvs_get_config(h)
    kb_ref, vb_ref = oracle_blocks(w, layer, n_tokens)
    P = -(-n_tokens // 256)
    for p in range(P):
        lo, hi = p * 256, min(n_tokens, (p + 1) * 256)
        kb, vb = export_page(h, cfg, layer, p, 0)
        assert np.array_equal(kb[: hi - lo], kb_ref[lo:hi]), f"host K blocks differ on page {p}"
        assert np.array_equal(vb[: hi - lo], vb_ref[lo:hi]), f"host V blocks differ on page {p}"
        kind, idx = kvs.kvs_page_location(h, layer, p)
        ok_kind, ok_idx = oracle.page_location(n_tokens, cfg.n_resident_pages, p)
        assert (kind, idx) == (ok_kind, ok_idx)
        if kind == kvs.KVS_PAGE_RESIDENT:
            kd, vd = export_page(h, cfg, layer, p, 1)
            assert np.array_equal(kd[: hi - lo], kb_ref[lo:hi]), f"resident K blocks differ on page {p}"
            assert np.array_equal(vd[: hi - lo], vb_ref[lo:hi]), f"resident V blocks differ on page {p}"


def test_append_blocks_bit_exact(kvs):
    w = small("append", n_q_heads=32, n_kv_heads=8, ctx=2600, n_resident_pages=4)
    cfg = make_cfg(w, max_q_tokens=256)
    h = kvs.kvs_create(cfg, 0)
    try:
        # ragged append widths, crossing page boundaries
        pos = 0
        for n in [1, 7, 255, 256, 1, 300, 513, 2, 1000, 265]:
            k, v = W.kv_tokens(w, 0, pos, pos + n)
            kvs.kvs_append(h, 0, pos, n, to_dev(k), to_dev(v))
            pos += n
        torch().cuda.synchronize()
        assert pos == 2600
        _check_pages(kvs, h, w, 0, pos)
    finally:
        kvs.kvs_destroy(h)


def test_append_special_values_bit_exact(kvs):
    """Zero rows, constant rows, ties of |x|, subnormals, extremes and rounding ties."""
    t = torch()
    H = 2
    rng = np.random.default_rng(3)
    rows = []
    rows.append(np.zeros((H, 128)))
    rows.append(np.full((H, 128), 0.75))
    rows.append(np.full((H, 128), -3.0))
    r = np.zeros((H, 128)); r[:, 0] = -1.0; r[:, 1] = 1.0; rows.append(r)      # |x| tie: first wins
    r = np.zeros((H, 128)); r[:, 5] = 1.0; r[:, 3] = -1.0; rows.append(r)
    rows.append(np.full((H, 128), 2.0 ** -24))                                     # subnormal fp16
    rows.append(rng.standard_normal((H, 128)) * 2.0 ** -20)
    rows.append(np.clip(rng.standard_normal((H, 128)) * 3e4, -65504, 65504))
    # exact Q8_0 rounding ties: amax 127/128 -> d = 1/128, x = k/256 with k odd
    r = np.tile(np.concatenate([[127 / 128], (np.arange(31) * 2 + 1) / 256.0 * np.where(np.arange(31) % 2, -1, 1)]), (H, 4)); rows.append(r)
    # exact Q4_0 boundaries: m = -1 -> d = 0.125, x = (k - 8.5)/8 boundaries
    r = np.tile(np.concatenate([[-1.0], (np.arange(31) % 16 - 8) / 8.0 + 1 / 16.0]), (H, 4)); rows.append(r)
    for _ in range(30):
        rows.append(rng.standard_normal((H, 128)) * np.where(rng.random((H, 128)) < 0.05, 8, 1))
    k = np.stack(rows).astype(np.float16)
    v = k[::-1].copy()
    n = k.shape[0]
    cfg = kvs.make_config(1, 8, H, 1024, n_resident_pages=4, n_ring_slots=0, max_q_tokens=64)
    h = kvs.kvs_create(cfg, 0)
    try:
        kvs.kvs_append(h, 0, 0, n, to_dev(k), to_dev(v))
        t.cuda.synchronize()
        kb_ref, vb_ref = oracle.quantize_rows(k, v)
        kb, vb = export_page(h, kvs.kvs_get_config(h), 0, 0, 0)
        assert np.array_equal(kb[:n], kb_ref)
        assert np.array_equal(vb[:n], vb_ref)
        kd, vd = export_page(h, kvs.kvs_get_config(h), 0, 0, 1)
        assert np.array_equal(kd[:n], kb_ref) and np.array_equal(vd[:n], vb_ref)
    finally:
        kvs.kvs_destroy(h)


# ---------------------------------------------------------------------------
# attention parity
# ---------------------------------------------------------------------------
def _run_and_check(kvs, w, cfg=None, layers=None):
    cfg = cfg or make_cfg(w)
    h = kvs.kvs_create(cfg, 0)
    try:
        for layer in (layers or range(w.n_layers)):
            prefill(h, w, layer, w.pos0)
            out, lse = step(h, w, layer, w.pos0, w.n_q)
            ref_out, ref_lse = oracle_step(w, layer, w.pos0, w.n_q)
            assert_close(out, lse, ref_out, ref_lse)
        return h
    finally:
        kvs.kvs_destroy(h)


def test_tiny_all_resident_decode_full_size(kvs):
    # the tiny workload at its full size: 1 layer, 8/2 heads, 4096 tokens, all resident
    _run_and_check(kvs, W.WORKLOADS["tiny_decode_4k"])


@pytest.mark.parametrize("ctx", [1, 200, 256, 257, 1500, 3000, 4097])
def test_decode_streamed_ragged(kvs, ctx):
    # 3 resident pages, ring of 4 slots in chunks of 2: several chunks and a ragged tail
    w = small(f"ragged{ctx}", ctx=ctx, n_resident_pages=3, n_ring_slots=4)
    _run_and_check(kvs, w)


@pytest.mark.parametrize("heads", [(32, 8), (40, 8), (8, 8), (16, 2)])
def test_decode_gqa_shapes(kvs, heads):
    w = small(f"gqa{heads}", n_q_heads=heads[0], n_kv_heads=heads[1], ctx=2300, n_layers=1)
    _run_and_check(kvs, w)


def test_decode_outliers(kvs):
    # the 32K workload's value mix (1 % of K/V elements x8) at a smaller context
    w = dataclasses.replace(W.WORKLOADS["streamed_decode_32k"], ctx=5000, n_layers=2,
                            n_resident_pages=8, n_ring_slots=8)
    _run_and_check(kvs, w)


@pytest.mark.parametrize("n_q,ctx", [(4, 3000), (4, 257), (2, 2), (16, 2000), (64, 1100), (256, 2048)])
def test_multi_token_causal(kvs, n_q, ctx):
    w = small(f"mt{n_q}", n_q=n_q, n_q_heads=40, n_kv_heads=8, ctx=ctx, n_resident_pages=3,
              n_ring_slots=4, n_layers=1)
    _run_and_check(kvs, w)


def test_streaming_equals_all_resident(kvs):
    t = torch()
    w = small("onoff", ctx=4000, n_layers=1, n_q_heads=32, n_kv_heads=8)
    res = {}
    for mode, over in {"stream": dict(n_resident_pages=2, n_ring_slots=4),
                       "resident": dict(n_resident_pages=16, n_ring_slots=0)}.items():
        cfg = make_cfg(w, **over)
        h = kvs.kvs_create(cfg, 0)
        try:
            prefill(h, w, 0, w.pos0)
            out, lse = step(h, w, 0, w.pos0, 1)
            pages = [export_page(h, kvs.kvs_get_config(h), 0, p, 0) for p in range(16)]
            res[mode] = (out, lse, pages)
        finally:
            kvs.kvs_destroy(h)
    for (ka, va), (kb, vb) in zip(res["stream"][2], res["resident"][2]):
        assert np.array_equal(ka, kb) and np.array_equal(va, vb)
    ref_out, ref_lse = oracle_step(w, 0, w.pos0, 1)
    for mode in res:
        assert_close(res[mode][0], res[mode][1], ref_out, ref_lse)
    np.testing.assert_allclose(res["stream"][0], res["resident"][0], rtol=0, atol=2e-5)


def test_rollback_and_reappend(kvs):
    """A rejected speculative draft: roll back over a page boundary and re-append."""
    t = torch()
    w = small("rb", ctx=2000, n_layers=1, n_resident_pages=2, n_ring_slots=4, n_q=4)
    w2 = dataclasses.replace(w, seed=99)  # different tokens for the re-append
    cfg = make_cfg(w, max_q_tokens=64)
    h = kvs.kvs_create(cfg, 0)
    try:
        prefill(h, w, 0, 1800)
        # roll back to 1530 (pages 5 and 6 drop out, page 4 re-enters the resident set)
        k2, v2 = W.kv_tokens(w2, 0, 1530, 1560)
        kvs.kvs_append(h, 0, 1530, 30, to_dev(k2), to_dev(v2))
        q = W.queries(w, 0, 1556, 4)
        out = t.empty((4, w.n_q_heads, 128), dtype=t.float32, device="cuda")
        lse = t.empty((4, w.n_q_heads), dtype=t.float32, device="cuda")
        kvs.kvs_attend(h, 0, 1556, 4, to_dev(q), out, lse)
        t.cuda.synchronize()
        assert kvs.kvs_layer_length(h, 0) == 1560
        k1, v1 = W.kv_tokens(w, 0, 0, 1530)
        kk = np.concatenate([k1, k2])
        vv = np.concatenate([v1, v2])
        kb, vb = oracle.quantize_rows(kk, vv)
        ref_out, ref_lse = oracle.attention(kb, vb, q, 1556)
        assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_out, ref_lse)
        cfg_r = kvs.kvs_get_config(h)
        for p in range(7):
            lo, hi = p * 256, min(1560, (p + 1) * 256)
            a, b = export_page(h, cfg_r, 0, p, 0)
            assert np.array_equal(a[: hi - lo], kb[lo:hi]) and np.array_equal(b[: hi - lo], vb[lo:hi])
            if kvs.kvs_page_location(h, 0, p)[0] == kvs.KVS_PAGE_RESIDENT:
                a, b = export_page(h, cfg_r, 0, p, 1)
                assert np.array_equal(a[: hi - lo], kb[lo:hi]) and np.array_equal(b[: hi - lo], vb[lo:hi])
    finally:
        kvs.kvs_destroy(h)


@pytest.mark.parametrize("mem", ["pinned", "pageable"])
@pytest.mark.parametrize("n_q,heads", [(1, (8, 2)), (4, (40, 8))])
def test_host_pointer_io(kvs, mem, n_q, heads):
    """Q/K/V/out/lse in host memory: pinned buffers cross PCIe inside the
    library's kernels, pageable ones through its staging buffers.  Either way
    the results are the bits the device-pointer calls give."""
    t = torch()
    w = small("hostio", ctx=1500, n_layers=1, n_q=n_q, n_q_heads=heads[0], n_kv_heads=heads[1])
    hd = kvs.kvs_create(make_cfg(w), 0)
    hh = kvs.kvs_create(make_cfg(w), 0)
    try:
        k, v = W.kv_tokens(w, 0, w.pos0, w.ctx)
        q = W.queries(w, 0, w.pos0, n_q)
        # device pointers
        prefill(hd, w, 0, w.pos0)
        out_d, lse_d = step(hd, w, 0, w.pos0, n_q)
        # host pointers
        prefill(hh, w, 0, w.pos0)
        if mem == "pinned":
            kh, vh, qh = (t.from_numpy(x).pin_memory() for x in (k, v, q))
            out = t.empty((n_q, w.n_q_heads, 128), dtype=t.float32).pin_memory()
            lse = t.empty((n_q, w.n_q_heads), dtype=t.float32).pin_memory()
        else:
            kh, vh, qh = (np.ascontiguousarray(x) for x in (k, v, q))
            out = t.from_numpy(np.zeros((n_q, w.n_q_heads, 128), np.float32))
            lse = t.from_numpy(np.zeros((n_q, w.n_q_heads), np.float32))
        kvs.kvs_append(hh, 0, w.pos0, n_q, kh, vh)
        kvs.kvs_attend(hh, 0, w.pos0, n_q, qh, out, lse)
        kvs.kvs_sync(hh, None, 30.0)
        assert np.array_equal(out.numpy(), out_d) and np.array_equal(lse.numpy(), lse_d)
        assert_close(out.numpy(), lse.numpy(), *oracle_step(w, 0, w.pos0, n_q))
    finally:
        kvs.kvs_destroy(hd)
        kvs.kvs_destroy(hh)


def test_repeated_steps_are_stable(kvs):
    """The benchmark's steady state: roll back one token and redo the step many times."""
    t = torch()
    w = small("steady", ctx=3000, n_layers=3, n_q_heads=32, n_kv_heads=8)
    cfg = make_cfg(w)
    h = kvs.kvs_create(cfg, 0)
    try:
        for layer in range(3):
            prefill(h, w, layer, w.pos0)
        outs = []
        for it in range(5):
            for layer in range(3):
                o, l = step(h, w, layer, w.pos0, 1)
                if layer == 1:
                    outs.append((o, l))
        for o, l in outs[1:]:
            assert np.array_equal(o, outs[0][0]) and np.array_equal(l, outs[0][1])
        ref_out, ref_lse = oracle_step(w, 1, w.pos0, 1)
        assert_close(outs[0][0], outs[0][1], ref_out, ref_lse)
    finally:
        kvs.kvs_destroy(h)
