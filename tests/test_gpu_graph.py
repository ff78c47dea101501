"""A whole decode step (append + attend for every layer) captured into a CUDA
graph and replayed: the ring's copy stream and the attention side streams
(resident, ring, in-place share) join the capture, and replays give the same
bits as plain calls before and after."""
import numpy as np
import pytest

from host_streamed_paged_kvs_b200 import workload as W
from kvs_testlib import assert_close, make_cfg, oracle_step, prefill, to_dev, torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_q,heads,pct", [(1, (32, 8), 0), (1, (32, 8), 80), (1, (32, 8), 100),
                                            (4, (40, 8), 0), (64, (40, 8), 0)])
def test_graph_captured_step_matches_plain_calls(n_q, heads, pct):
    t = torch()
    from host_streamed_paged_kvs_b200 import kvs
    w = W.Workload("graph", n_layers=3, n_q=n_q, n_q_heads=heads[0], n_kv_heads=heads[1], ctx=3000,
                   n_resident_pages=3, n_ring_slots=4, seed=31)
    h = kvs.kvs_create(make_cfg(w, zero_copy_pct=pct), 0)
    s = t.cuda.Stream()
    try:
        for layer in range(w.n_layers):
            prefill(h, w, layer, w.pos0)
        ks, vs, qs = [], [], []
        for layer in range(w.n_layers):
            k, v = W.kv_tokens(w, layer, w.pos0, w.ctx)
            ks.append(to_dev(k)); vs.append(to_dev(v)); qs.append(to_dev(W.queries(w, layer, w.pos0)))
        out = t.zeros((w.n_layers, n_q, w.n_q_heads, 128), dtype=t.float32, device="cuda")
        lse = t.zeros((w.n_layers, n_q, w.n_q_heads), dtype=t.float32, device="cuda")

        def step():
            for layer in range(w.n_layers):
                kvs.kvs_append(h, layer, w.pos0, n_q, ks[layer], vs[layer], s)
                kvs.kvs_attend(h, layer, w.pos0, n_q, qs[layer], out[layer], lse[layer], s)

        t.cuda.synchronize()
        with t.cuda.stream(s):
            step()
        s.synchronize()
        plain = (out.clone(), lse.clone())

        g = t.cuda.CUDAGraph()
        out.zero_(); lse.zero_()
        t.cuda.synchronize()
        with t.cuda.graph(g, stream=s):
            step()
        for _ in range(3):
            out.zero_(); lse.zero_()
            g.replay()
            t.cuda.synchronize()
            assert t.equal(out, plain[0]) and t.equal(lse, plain[1])

        # plain calls after the replays still agree
        out.zero_(); lse.zero_()
        t.cuda.synchronize()
        with t.cuda.stream(s):
            step()
        s.synchronize()
        assert t.equal(out, plain[0]) and t.equal(lse, plain[1])
        ref = oracle_step(w, 2, w.pos0, n_q)
        assert_close(out[2].cpu().numpy(), lse[2].cpu().numpy(), *ref)
        del g
    finally:
        t.cuda.synchronize()
        kvs.kvs_destroy(h)


def test_graph_of_appends_only():
    # The copy stream joins a capture at its first append; a capture that holds
    # appends only must still end (every stream joined back) and replay, and
    # attention after it sees the appended tokens.
    t = torch()
    from host_streamed_paged_kvs_b200 import kvs
    w = W.Workload("graph_appends", n_layers=3, n_q=4, n_q_heads=40, n_kv_heads=8, ctx=3000,
                   n_resident_pages=3, n_ring_slots=4, seed=32)
    h = kvs.kvs_create(make_cfg(w), 0)
    s = t.cuda.Stream()
    try:
        for layer in range(w.n_layers):
            prefill(h, w, layer, w.pos0)
        ks, vs = [], []
        for layer in range(w.n_layers):
            k, v = W.kv_tokens(w, layer, w.pos0, w.ctx)
            ks.append(to_dev(k)); vs.append(to_dev(v))
        t.cuda.synchronize()
        g = t.cuda.CUDAGraph()
        with t.cuda.graph(g, stream=s):
            for layer in range(w.n_layers):
                kvs.kvs_append(h, layer, w.pos0, w.n_q, ks[layer], vs[layer], s)
        for _ in range(2):
            g.replay()
        t.cuda.synchronize()
        del g
        q = to_dev(W.queries(w, 2, w.pos0))
        out = t.zeros((w.n_q, w.n_q_heads, 128), dtype=t.float32, device="cuda")
        lse = t.zeros((w.n_q, w.n_q_heads), dtype=t.float32, device="cuda")
        with t.cuda.stream(s):
            kvs.kvs_attend(h, 2, w.pos0, w.n_q, q, out, lse, s)
        s.synchronize()
        assert_close(out.cpu().numpy(), lse.cpu().numpy(), *oracle_step(w, 2, w.pos0, w.n_q))
    finally:
        t.cuda.synchronize()
        kvs.kvs_destroy(h)
