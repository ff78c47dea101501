"""The bench's copy/compute timeline summary, on a hand-made trace (host
logic only): copy-engine busy time, overlap with kernels, link busy time and
the gaps between link activity."""
import json

import bench


def test_timeline_summary_on_a_hand_made_trace(tmp_path):
    # 0..100 us window: copies [0,10) and [20,40) (2 MB each); an in-place
    # decode launch [35,60); a TMA decode launch [5,25); a merge [95,100)
    ev = [
        {"ph": "X", "cat": "gpu_memcpy", "name": "Memcpy HtoD (Pinned -> Device)", "ts": 0, "dur": 10,
         "args": {"bytes": 2e6}},
        {"ph": "X", "cat": "gpu_memcpy", "name": "Memcpy HtoD (Pinned -> Device)", "ts": 20, "dur": 20,
         "args": {"bytes": 2e6}},
        {"ph": "X", "cat": "gpu_memcpy", "name": "Memcpy DtoH (Device -> Pinned)", "ts": 60, "dur": 5,
         "args": {"bytes": 1e3}},
        {"ph": "X", "cat": "kernel", "name": "void kvs::decode_kernel<1, true, 2>(kvs::DecodeArgs, CUtensorMap)",
         "ts": 35, "dur": 25, "args": {"stream": 7}},
        {"ph": "X", "cat": "kernel", "name": "void kvs::decode_kernel<1, false, 2>(kvs::DecodeArgs, CUtensorMap)",
         "ts": 5, "dur": 20, "args": {"stream": 9}},
        {"ph": "X", "cat": "kernel", "name": "kvs::merge_kernel(kvs::MergeArgs)", "ts": 95, "dur": 5,
         "args": {"stream": 3}},
        {"ph": "i", "name": "marker", "ts": 50},
    ]
    p = tmp_path / "t.json"
    p.write_text(json.dumps({"traceEvents": ev}))
    s = bench.timeline_summary(str(p), 2, 55.0)
    assert s["window_us"] == 100 and s["us_per_step"] == 50
    assert s["h2d_copies"] == 2 and s["h2d_copy_bytes"] == 4e6
    assert s["copy_engine_busy_us"] == 30 and abs(s["copy_engine_busy_frac"] - 0.3) < 1e-12
    assert abs(s["copy_gbs_while_busy"] - 4e6 / 30e-6 / 1e9) < 1e-9
    # copy time under kernels: [5,10) and [20,25) and [35,40) = 15 of 30
    assert abs(s["copy_time_overlapping_kernels_frac"] - 0.5) < 1e-12
    # link: copies and in-place launches: [0,10) [20,60) = 50 of 100; gap 10
    assert abs(s["link_busy_frac"] - 0.5) < 1e-12
    assert s["largest_link_gaps_us"] == [10]
    assert s["kernel_launches"] == {"decode_in_place": 1, "decode_tma": 1, "merge_kernel": 1}
    assert s["kernel_busy_us"]["decode_in_place"] == 25


def test_interval_helpers():
    u = bench._union([(5, 7), (0, 2), (1, 3), (7, 8)])
    assert u == [[0, 3], [5, 8]]
    assert bench._length(u) == 6
    assert bench._intersect(u, [[2, 6]]) == 2
