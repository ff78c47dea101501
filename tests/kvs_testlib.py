"""Helpers shared by the GPU tests: drive libkvs through its binding and build
the oracle's expected values from the same seeded inputs."""
from __future__ import annotations

import numpy as np

import oracle
from host_streamed_paged_kvs_b200 import workload as W

D = 128
T = 256
# tolerance of the float outputs against the binary64 oracle
O_RTOL_ABS = 1e-3   # |out - ref| <= 1e-3 * (1 + |ref|)
LSE_ATOL = 1e-4     # |lse - ref| <= 1e-4


def torch():
    import torch as _t
    return _t


def make_cfg(w: W.Workload, max_q_tokens=None, **over):
    from host_streamed_paged_kvs_b200 import kvs
    args = dict(n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                max_ctx=w.ctx, n_resident_pages=w.n_resident_pages,
                n_ring_slots=w.n_ring_slots,
                max_q_tokens=max_q_tokens if max_q_tokens is not None else w.n_q)
    args.update(over)
    return kvs.make_config(**args)


def to_dev(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a)).cuda()


def prefill(h, w: W.Workload, layer: int, upto: int, chunk: int = 16384, stream=None):
    """Append tokens [0, upto) of `layer` through kvs_append (device K/V)."""
    from host_streamed_paged_kvs_b200 import kvs
    pos = 0
    while pos < upto:
        n = min(chunk, upto - pos)
        k, v = W.kv_tokens(w, layer, pos, pos + n)
        kvs.kvs_append(h, layer, pos, n, to_dev(k), to_dev(v), stream)
        pos += n


def step(h, w: W.Workload, layer: int, pos0: int, n_q: int, stream=None):
    """Append the step's n_q tokens at pos0 and attend; returns (out, lse) as numpy."""
    from host_streamed_paged_kvs_b200 import kvs
    t = torch()
    k, v = W.kv_tokens(w, layer, pos0, pos0 + n_q)
    q = W.queries(w, layer, pos0, n_q)
    kvs.kvs_append(h, layer, pos0, n_q, to_dev(k), to_dev(v), stream)
    out = t.empty((n_q, w.n_q_heads, D), dtype=t.float32, device="cuda")
    lse = t.empty((n_q, w.n_q_heads), dtype=t.float32, device="cuda")
    kvs.kvs_attend(h, layer, pos0, n_q, to_dev(q), out, lse, stream)
    t.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def oracle_blocks(w: W.Workload, layer: int, upto: int, v_type: int = oracle.V_Q4_0,
                  k_type: int = oracle.K_Q8_0):
    k, v = W.kv_tokens(w, layer, 0, upto)
    return oracle.quantize_rows(k, v, v_type, k_type)


def oracle_step(w: W.Workload, layer: int, pos0: int, n_q: int, rows=None, v_type: int = oracle.V_Q4_0,
                k_type: int = oracle.K_Q8_0):
    """Oracle out/lse for the step's queries over the layer's history [0, pos0+n_q)."""
    kb, vb = oracle_blocks(w, layer, pos0 + n_q, v_type, k_type)
    q = W.queries(w, layer, pos0, n_q)
    return oracle.attention(kb, vb, q, pos0, v_type, k_type)


def assert_close(out, lse, ref_out, ref_lse):
    err = np.abs(out.astype(np.float64) - ref_out)
    bound = O_RTOL_ABS * (1.0 + np.abs(ref_out))
    worst = float((err / bound).max())
    assert np.all(err <= bound), f"out mismatch: worst err/bound = {worst:.3g}, max err {err.max():.3g}"
    lerr = np.abs(lse.astype(np.float64) - ref_lse)
    assert np.all(lerr <= LSE_ATOL), f"lse mismatch: max err {lerr.max():.3g}"
    return worst, float(lerr.max())


def export_page(h, cfg, layer, page, from_device):
    from host_streamed_paged_kvs_b200 import kvs
    H = cfg.n_kv_heads
    vbytes = {kvs.KVS_TYPE_Q8_0: 34, kvs.KVS_TYPE_Q5_0: 22, kvs.KVS_TYPE_Q4_1: 20,
              kvs.KVS_TYPE_Q5_1: 24, kvs.KVS_TYPE_F16: 64}.get(cfg.type_v, 18)
    kbytes = 64 if cfg.type_k == kvs.KVS_TYPE_F16 else 34
    nk = T * H * 4 * kbytes
    nv = T * H * 4 * vbytes
    buf = np.zeros(nk + nv, np.uint8)
    kvs.kvs_export_page(h, layer, page, from_device, buf)
    kb = buf[:nk].reshape(T, H, 4, kbytes)
    vb = buf[nk:].reshape(T, H, 4, vbytes)
    return kb, vb
