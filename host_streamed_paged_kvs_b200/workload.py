"""Seeded synthetic workloads: shapes and the random fp16 inputs they use.

This module holds no arithmetic of the attention method itself.  It only
describes the workload shapes and draws the seeded fp16 Q/K/V inputs, so the
CUDA path and the CPU oracle can be fed identical data.

Inputs are drawn page by page (256 tokens) from ``numpy.random.default_rng``
seeded with ``[seed, layer, page]``; any page can therefore be regenerated
independently of the others, which lets a sampled check rebuild one layer's
history without the rest.  Values are N(0, 1) rounded to fp16; the 32K
streamed-decode workload multiplies a Bernoulli(0.01) subset of the K/V
elements by 8 (outliers).
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

PAGE_TOKENS = 256
HEAD_DIM = 128
_Q_STREAM = 1 << 30  # SeedSequence word that separates query draws from K/V pages


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_q: int              # query tokens per step (1 decode, 4 verify, 256 prefill chunk)
    n_q_heads: int
    n_kv_heads: int
    ctx: int              # tokens attended by the last query of a step
    n_resident_pages: int  # 0 = auto rule
    n_ring_slots: int
    seed: int
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    head_dim: int = HEAD_DIM
    page_tokens: int = PAGE_TOKENS
    type_v: int = 2       # V type: 1 F16, 2 Q4_0, 3 Q4_1, 6 Q5_0, 7 Q5_1, 8 Q8_0 (the q8_0/q8_0 pair)

    @property
    def n_pages(self) -> int:
        return (self.ctx + self.page_tokens - 1) // self.page_tokens

    @property
    def pos0(self) -> int:
        """Position of the first query token of the timed step."""
        return self.ctx - self.n_q

    def scaled(self, ctx: int, n_layers: Optional[int] = None, n_resident_pages: Optional[int] = None,
               n_ring_slots: Optional[int] = None, name: Optional[str] = None) -> "Workload":
        """Same shape family at a smaller context (for parity runs)."""
        return dataclasses.replace(
            self, name=name or f"{self.name}@{ctx}", ctx=ctx,
            n_layers=self.n_layers if n_layers is None else n_layers,
            n_resident_pages=self.n_resident_pages if n_resident_pages is None else n_resident_pages,
            n_ring_slots=self.n_ring_slots if n_ring_slots is None else n_ring_slots)


# The five workloads of the method's evaluation: tiny all-resident decode, 32K
# streamed decode, 256K long-context decode (auto resident set = 103 pages),
# speculative verify over a 17-layer pool, and a 256-token prefill chunk.
WORKLOADS = {
    "tiny_decode_4k": Workload("tiny_decode_4k", n_layers=1, n_q=1, n_q_heads=8, n_kv_heads=2,
                               ctx=4096, n_resident_pages=16, n_ring_slots=0, seed=0),
    "streamed_decode_32k": Workload("streamed_decode_32k", n_layers=16, n_q=1, n_q_heads=32,
                                    n_kv_heads=8, ctx=32768, n_resident_pages=64, n_ring_slots=8,
                                    seed=1, outlier_frac=0.01, outlier_scale=8.0),
    "long_decode_256k": Workload("long_decode_256k", n_layers=16, n_q=1, n_q_heads=40,
                                 n_kv_heads=8, ctx=262144, n_resident_pages=0, n_ring_slots=16,
                                 seed=2),
    "verify_128k": Workload("verify_128k", n_layers=17, n_q=4, n_q_heads=40, n_kv_heads=8,
                            ctx=131072, n_resident_pages=178, n_ring_slots=16, seed=3),
    "prefill_chunk_64k": Workload("prefill_chunk_64k", n_layers=1, n_q=256, n_q_heads=40,
                                  n_kv_heads=8, ctx=65536, n_resident_pages=64, n_ring_slots=16,
                                  seed=4),
    # the 32K streamed decode with the q8_0/q8_0 pair (V as Q8_0: 2176 B per token per layer)
    "streamed_decode_32k_q8v": Workload("streamed_decode_32k_q8v", n_layers=16, n_q=1, n_q_heads=32,
                                        n_kv_heads=8, ctx=32768, n_resident_pages=64, n_ring_slots=8,
                                        seed=5, outlier_frac=0.01, outlier_scale=8.0, type_v=8),
    # the same with V as Q5_0 (1728 B per token per layer)
    "streamed_decode_32k_q5v": Workload("streamed_decode_32k_q5v", n_layers=16, n_q=1, n_q_heads=32,
                                        n_kv_heads=8, ctx=32768, n_resident_pages=64, n_ring_slots=8,
                                        seed=6, outlier_frac=0.01, outlier_scale=8.0, type_v=6),
    # V as Q4_1 / Q5_1 (1728 / 1856 B per token per layer)
    "streamed_decode_32k_q41v": Workload("streamed_decode_32k_q41v", n_layers=16, n_q=1, n_q_heads=32,
                                         n_kv_heads=8, ctx=32768, n_resident_pages=64, n_ring_slots=8,
                                         seed=7, outlier_frac=0.01, outlier_scale=8.0, type_v=3),
    "streamed_decode_32k_q51v": Workload("streamed_decode_32k_q51v", n_layers=16, n_q=1, n_q_heads=32,
                                         n_kv_heads=8, ctx=32768, n_resident_pages=64, n_ring_slots=8,
                                         seed=8, outlier_frac=0.01, outlier_scale=8.0, type_v=7),
}
# The bench's default is the largest single-GPU decode configuration: 256K
# context, where most of every step streams from host memory.
DEFAULT_BENCH = "long_decode_256k"
# Share (%) of a decode step's streamed pages that the decode kernel reads in
# place from the mapped pinned history while the copy engine brings the rest
# through the ring: in-place reads pay no per-copy cost, and the ring keeps
# copying ahead into the next layer.  Tuned on the 32K streamed decode
# workload (70-90 % within noise of each other, ring-only 4 % slower).
ZERO_COPY_PCT = 80
# The same share for the wider calls of the tensor-core path (verify batches,
# prefill chunks), whose in-place launch holds about 120 of the 148 SMs.
# Measured on the verify workload, in place only (100) ran 3 % slower than the
# ring alone and shares of 30-70 % were no faster (8-page ring copies are as
# fast as the link allows); on the prefill chunk every tile pair of a kv head
# reads the host pages itself, five times the PCIe bytes, so the ring alone (0)
# is the default.
ZERO_COPY_PCT_WIDE = 0


def _page_kv(w: Workload, layer: int, page: int):
    rng = np.random.default_rng([w.seed, layer, page])
    shape = (w.page_tokens, w.n_kv_heads, w.head_dim)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    if w.outlier_frac > 0:
        k = np.where(rng.random(shape, dtype=np.float32) < w.outlier_frac, k * w.outlier_scale, k)
        v = np.where(rng.random(shape, dtype=np.float32) < w.outlier_frac, v * w.outlier_scale, v)
    return k.astype(np.float16), v.astype(np.float16)


def kv_tokens(w: Workload, layer: int, t0: int, t1: int, threads: int = 0):
    """fp16 K, V for tokens [t0, t1) of `layer`: arrays [t1-t0, n_kv_heads, head_dim]."""
    T = w.page_tokens
    p0, p1 = t0 // T, (t1 + T - 1) // T
    pages = list(range(p0, p1))
    threads = threads or min(16, os.cpu_count() or 1)
    if len(pages) > 2 and threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(lambda p: _page_kv(w, layer, p), pages))
    else:
        parts = [_page_kv(w, layer, p) for p in pages]
    k = np.concatenate([a for a, _ in parts], axis=0)
    v = np.concatenate([b for _, b in parts], axis=0)
    lo = t0 - p0 * T
    return (np.ascontiguousarray(k[lo:lo + (t1 - t0)]),
            np.ascontiguousarray(v[lo:lo + (t1 - t0)]))


def queries(w: Workload, layer: int, pos0: int, n_q: Optional[int] = None):
    """fp16 Q [n_q, n_q_heads, head_dim] for the step whose first query sits at pos0."""
    n_q = w.n_q if n_q is None else n_q
    rng = np.random.default_rng([w.seed, layer, _Q_STREAM, pos0])
    q = rng.standard_normal((n_q, w.n_q_heads, w.head_dim), dtype=np.float32)
    return q.astype(np.float16)
