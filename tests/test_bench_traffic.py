"""The bench's per-launch DRAM/PCIe traffic figures (host logic only): a
capture's bytes per page applied to the pages another launch reads, the
guards on workload, page format and kernel source."""
import dataclasses

import bench
from host_streamed_paged_kvs_b200 import workload as W

PB = 425984  # bytes per page of the q8_0 K / q4_0 V format, 8 kv heads


def _sha_ok(kernel):
    return bench._ncu_entry(kernel, W.WORKLOADS[bench.NCU_TRAFFIC[kernel]["workload"]], True) is not None


def test_decode_traffic_scales_by_pages_to_another_workload():
    if not _sha_ok("decode_kernel"):
        return  # kernel changed since the capture: the bench reports null, checked below
    t = bench.NCU_TRAFFIC["decode_kernel"]
    w = W.WORKLOADS["long_decode_256k"]
    # one resident launch of 103 pages and two ring launches of 8 pages
    got = bench.ncu_traffic("decode_kernel", w, PB, 103 * PB, 16 * PB, 3)
    want = (t["resident"][0] / t["resident"][1] * 103 + t["ring"][0] / t["ring"][1] * 16) / 3
    assert abs(got - want) < 1e-6 * want
    # the captured launches read their pages once: within 2 % of the page bytes
    assert 1.0 <= got / ((103 + 16) * PB / 3) < 1.02
    pcie = bench.ncu_in_place(w, PB, "pcie", 737)
    assert abs(pcie - t["in_place_pcie"][0] / t["in_place_pcie"][1] * 737) < 1
    assert bench.ncu_in_place(w, PB, "dram", 737) == t["in_place"][0]


def test_traffic_guards():
    w = W.WORKLOADS["long_decode_256k"]
    # another page format: no figure
    assert bench.ncu_traffic("decode_kernel", dataclasses.replace(w, type_v=8), PB, PB, PB, 2) is None
    # the tensor-core kernel's figures hold for the captured workload only
    assert bench.ncu_traffic("chunk_mma_kernel", W.WORKLOADS["verify_128k"], PB, PB, PB, 2) is None
    # no launches: no figure
    assert bench.ncu_traffic("decode_kernel", w, PB, 0, 0, 0) is None


def test_traffic_is_null_once_the_source_changes(monkeypatch):
    e = dict(bench.NCU_TRAFFIC["decode_kernel"], sha="0000000000000000")
    monkeypatch.setitem(bench.NCU_TRAFFIC, "decode_kernel", e)
    w = W.WORKLOADS["streamed_decode_32k"]
    assert bench.ncu_traffic("decode_kernel", w, PB, 64 * PB, 4 * PB, 2) is None
    assert bench.ncu_in_place(w, PB, "pcie", 51) is None
