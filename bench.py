"""Benchmark: streamed decode-attention KV tokens/s/layer on B200, and its
fraction of the max(resident bytes / HBM BW, streamed bytes / H2D BW) roofline.

One step = one pass of the whole path over every layer of the workload:
quantize-on-append of the step's tokens (rolled back to the same position each
step, the steady state of a decode loop) and attention over the full history
(resident pages in place, older pages streamed from pinned host memory through
the copy-engine ring, split partials merged by log-sum-exp).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  With N > 1 (torchrun) every rank runs an
independent replica on its own GPU ("replicas only": the path has no exchange
step); value = all ranks' tokens / the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from host_streamed_paged_kvs_b200 import workload as W  # noqa: E402

METRIC = "streamed decode-attn KV tokens/s/layer; % of max(HBM,H2D) roofline, 1xB200"
UNIT = "KV tokens/s/layer"


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the launches
# captured with ncu and summarized under profiles/, as (bytes, pages the launch
# attended).  A launch of another size is scaled by its pages (the traffic of
# these launches grows with the pages they read); the decode kernel's figures
# serve every workload with the captured page format, the tensor-core kernel's
# only the captured workload (its re-reads depend on the query tiles).  A
# figure is used only while the kernel source is unchanged (sha256 prefix of
# the .cu file); otherwise traffic is reported as null.
NCU_TRAFFIC = {
    "decode_kernel": {"src": "kvs_kernels.cu", "sha": "fa1a72c4e1cd72cf",
                      "workload": "streamed_decode_32k", "type_v": 2,
                      "resident": (27297280, 64), "ring": (1737472, 4),
                      # in-place launch: DRAM bytes (Q and split records; they do not grow
                      # with the pages), and host-memory bytes read over PCIe
                      "in_place": (86272, 51), "in_place_pcie": (23763968, 51)},
    "chunk_mma_kernel": {"src": "kvs_chunk_mma.cu", "sha": "18d03cf82c7cfd65",
                         "workload": "prefill_chunk_64k", "type_v": 2,
                         "resident": (21223680, 6), "ring": (6100480, 8)},
}


def _ncu_entry(kernel: str, w, same_workload: bool):
    import hashlib
    t = NCU_TRAFFIC.get(kernel)
    if not t or t["type_v"] != w.type_v or (same_workload and t["workload"] != w.name):
        return None
    path = os.path.join(ROOT, "host_streamed_paged_kvs_b200", "csrc", t["src"])
    with open(path, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != t["sha"]:
            return None
    return t


def ncu_traffic(kernel: str, w, page_bytes: int, res_bytes: float, ring_bytes: float, n_launches: int):
    """Average DRAM traffic of one launch: the captured bytes per page of the
    resident and ring launches applied to the page bytes these launches read."""
    t = _ncu_entry(kernel, w, same_workload=(kernel != "decode_kernel"))
    if t is None or n_launches == 0:
        return None
    per_page = {k: t[k][0] / (t[k][1] * page_bytes) for k in ("resident", "ring")}
    return (per_page["resident"] * res_bytes + per_page["ring"] * ring_bytes) / n_launches


def ncu_in_place(w, page_bytes: int, field: str, pages_per_launch: float):
    """Traffic of one in-place decode launch: its DRAM bytes as captured, or its
    PCIe reads scaled by the pages it reads."""
    t = _ncu_entry("decode_kernel", w, same_workload=False)
    if t is None:
        return None
    if field == "dram":
        return t["in_place"][0]
    b, n = t["in_place_pcie"]
    return b / n * pages_per_launch


def best_big_copy_gbs(torch, dev, reps: int = 10) -> float:
    """Best host-to-device rate (GB/s) over `reps` transfers of 1 GiB from
    pinned memory in 64 MiB copies: the link's bound for the step roofline."""
    big = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
    dbig = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    best = 0.0
    cs = torch.cuda.Stream(device=dev)
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(cs)
        with torch.cuda.stream(cs):
            for i in range(16):
                dbig[i << 26:(i + 1) << 26].copy_(big[i << 26:(i + 1) << 26], non_blocking=True)
        b.record(cs)
        cs.synchronize()
        best = max(best, (1 << 30) / (a.elapsed_time(b) * 1e-3) / 1e9)
    del big, dbig
    return best


def reduce_max(x: float, dist=None, device=None) -> float:
    """Max of a per-rank time over all ranks (no-op for a single process)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, ctx: int, n_layers: int, ms_step: float) -> float:
    """Whole-job KV tokens attended per second per layer: every replica attends
    ctx tokens in each of its n_layers layers per step; the job's step time is
    the slowest replica's."""
    return world * ctx * n_layers / (ms_step * 1e-3)


def peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        self.f.close()
        os.unlink(self.f.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_layer_step(w: W.Workload, layer: int = 0, prepared=None):
    """Time the oracle on one layer's step of the workload: quantize the step's
    tokens and attend over the whole history.  Returns (seconds, prepared)."""
    import oracle
    if prepared is None:
        k, v = W.kv_tokens(w, layer, 0, w.pos0)
        kb, vb = oracle.quantize_rows(k, v, w.type_v)
        ks, vs = W.kv_tokens(w, layer, w.pos0, w.ctx)
        q = W.queries(w, layer, w.pos0)
        prepared = (kb, vb, ks, vs, q)
    kb, vb, ks, vs, q = prepared
    t0 = time.perf_counter()
    kbs, vbs = oracle.quantize_rows(ks, vs, w.type_v)
    kall = np.concatenate([kb, kbs])
    vall = np.concatenate([vb, vbs])
    oracle.attention(kall, vall, q, w.pos0, w.type_v)
    return time.perf_counter() - t0, prepared


def oracle_step_threaded(w: W.Workload, prepared, threads: int) -> float:
    """Wall time of the oracle over a whole step's attention, the (layer, kv
    head) problems spread over `threads` threads (the C oracle runs without the
    GIL).  Every layer reuses the prepared layer's data: the same work per layer."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    kb, vb, ks, vs, q = prepared
    G = w.n_q_heads // w.n_kv_heads
    t0 = time.perf_counter()
    kbs, vbs = oracle.quantize_rows(ks, vs, w.type_v)
    kall = np.concatenate([kb, kbs])
    vall = np.concatenate([vb, vbs])
    parts = [(np.ascontiguousarray(kall[:, g:g + 1]), np.ascontiguousarray(vall[:, g:g + 1]),
              np.ascontiguousarray(q[:, g * G:(g + 1) * G])) for g in range(w.n_kv_heads)]
    jobs = [parts[g] for _ in range(w.n_layers) for g in range(w.n_kv_heads)]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda p: oracle.attention(p[0], p[1], p[2], w.pos0, w.type_v), jobs))
    return time.perf_counter() - t0


def cpu_baseline(w: W.Workload, budget_s: float = 15.0):
    secs, prep = oracle_layer_step(w)
    times = [secs]
    while sum(times) < budget_s and len(times) < 8:
        t, _ = oracle_layer_step(w, prepared=prep)
        times.append(t)
    per_layer = statistics.median(times)
    threads = min(os.cpu_count() or 1, w.n_layers * w.n_kv_heads)
    threaded = None
    # all cores, only when one threaded step stays within the budget
    if per_layer * w.n_layers / threads < budget_s:
        ts = oracle_step_threaded(w, prep, threads)
        threaded = {"value": w.ctx * w.n_layers / ts, "unit": UNIT, "threads": threads,
                    "sample": f"one whole step of {w.name}: {w.n_layers} layers x {w.n_kv_heads} kv heads "
                              f"as independent oracle calls on a pool of {threads} threads"}
    return {"value": w.ctx / per_layer, "unit": UNIT, "cores": 1, "kind": "oracle",
            "all_cores": threaded,
            "sample": f"{len(times)} x one layer's step of {w.name} (append {w.n_q} token(s), "
                      f"binary64 attention of {w.n_q}x{w.n_q_heads} query rows over {w.ctx} keys), "
                      f"single thread, median {per_layer:.2f} s"}


def run_reference(args, w: W.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    _, prep = oracle_layer_step(w)
    for i in range(args.warmup + args.steps):
        t, _ = oracle_layer_step(w, prepared=prep)
        if i >= args.warmup:
            times.append(t)
    per = statistics.median(times)
    value = w.ctx / per
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "ctx": w.ctx, "n_layers_timed": 1,
                       "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "n_q": w.n_q},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step = one layer's step of {w.name} on the CPU oracle "
                                       f"(single thread)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# copy / compute timeline (CUPTI activity records through torch.profiler)
# ---------------------------------------------------------------------------
def _union(iv):
    """Merged [start, end) intervals of a list of (start, end)."""
    out = []
    for a, b in sorted(iv):
        if out and a <= out[-1][1]:
            out[-1][1] = max(out[-1][1], b)
        else:
            out.append([a, b])
    return out


def _length(iv):
    return sum(b - a for a, b in iv)


def _intersect(x, y):
    """Total length of the intersection of two merged interval lists."""
    i = j = 0
    tot = 0.0
    while i < len(x) and j < len(y):
        a, b = max(x[i][0], y[j][0]), min(x[i][1], y[j][1])
        if b > a:
            tot += b - a
        if x[i][1] < y[j][1]:
            i += 1
        else:
            j += 1
    return tot


def timeline_summary(trace_path: str, n_steps: int, h2d_peak: float):
    """Summary of one profiled run of n_steps steps from its trace: the
    host-to-device copy rows (the ring's copy engine), the library's kernels
    per kind, how much of the copy time overlaps kernels, and how busy the
    host-to-device link is (ring copies together with the in-place decode
    launches, which read host memory over the same link)."""
    with open(trace_path) as f:
        ev = json.load(f)["traceEvents"]
    kern, copies = [], []
    for e in ev:
        if e.get("ph") != "X":
            continue
        cat = e.get("cat", "")
        if cat == "kernel":
            kern.append(e)
        elif cat == "gpu_memcpy" and "HtoD" in e.get("name", ""):
            copies.append(e)
    if not kern:
        return None

    def kind(name):
        if "decode_kernel" in name:
            return "decode_in_place" if ", true," in name else "decode_tma"
        for k in ("chunk_mma_kernel", "merge_rows_kernel", "merge_kernel", "append_kernel", "copy16_kernel"):
            if k in name:
                return k
        return "other"

    t0 = min(e["ts"] for e in kern + copies)
    t1 = max(e["ts"] + e["dur"] for e in kern + copies)
    win = t1 - t0
    cp = _union([(e["ts"], e["ts"] + e["dur"]) for e in copies])
    kinds = {}
    for e in kern:
        kinds.setdefault(kind(e["name"]), []).append((e["ts"], e["ts"] + e["dur"]))
    all_k = _union([iv for v in kinds.values() for iv in v])
    zc = _union(kinds.get("decode_in_place", []))
    link = _union(cp + zc)
    gaps = sorted((b[0] - a[1] for a, b in zip(link, link[1:])), reverse=True)
    cbytes = sum(float(e.get("args", {}).get("bytes", 0)) for e in copies)
    streams = sorted({(e.get("args", {}).get("stream"), kind(e["name"])) for e in kern}, key=str)
    return {
        "steps": n_steps, "window_us": win, "us_per_step": win / n_steps,
        "h2d_copies": len(copies), "h2d_copy_bytes": cbytes,
        "copy_engine_busy_us": _length(cp), "copy_engine_busy_frac": _length(cp) / win,
        "copy_gbs_while_busy": cbytes / (_length(cp) * 1e-6) / 1e9 if cp else None,
        "copy_time_overlapping_kernels_frac": _intersect(cp, all_k) / _length(cp) if cp else None,
        "link_busy_frac": _length(link) / win,
        "link_busy_note": "union of ring copies and in-place decode launches (both read host memory over PCIe)",
        "largest_link_gaps_us": gaps[:5],
        "kernel_busy_us": {k: _length(_union(v)) for k, v in kinds.items()},
        "kernel_launches": {k: len(v) for k, v in kinds.items()},
        "streams_by_kind": [f"{st}:{k}" for st, k in streams],
        "h2d_gbs_peak_measured": h2d_peak,
    }


def capture_timeline(step_fn, n_steps: int, path: str, sync):
    """Record n_steps calls of step_fn under torch.profiler (CUPTI activity
    records of every kernel and copy, the library's included) and write the
    Chrome trace to path."""
    import torch
    from torch.profiler import ProfilerActivity, profile
    sync()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(n_steps):
            step_fn()
        sync()
    prof.export_chrome_trace(path)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
def run_gpu(args, w: W.Workload):
    import torch
    import torch.distributed as dist
    from host_streamed_paged_kvs_b200 import kvs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=600))
    dev = torch.device("cuda", local)

    L = w.n_layers
    # steps with streamed pages can read a share of them in place: the decode
    # share for decode widths, the wide share for the tensor-core path
    r0 = kvs.kvs_resolve_config(kvs.make_config(L, w.n_q_heads, w.n_kv_heads, w.ctx,
                                                n_resident_pages=w.n_resident_pages,
                                                n_ring_slots=w.n_ring_slots, type_v=w.type_v))[0]
    wide = w.n_q * (w.n_q_heads // w.n_kv_heads) > 8
    zc_able = r0.n_resident_pages < w.n_pages and w.n_ring_slots > 0
    tuned = W.ZERO_COPY_PCT_WIDE if wide else W.ZERO_COPY_PCT
    zc_pct = (tuned if args.zero_copy_pct < 0 else args.zero_copy_pct) if zc_able else 0
    zc_pct_wide = zc_pct if wide else 0
    cfg = kvs.make_config(L, w.n_q_heads, w.n_kv_heads, w.ctx, n_resident_pages=w.n_resident_pages,
                          n_ring_slots=w.n_ring_slots, max_q_tokens=w.n_q,
                          chunk_pages=args.chunk_pages, zero_copy_pct=0 if wide else zc_pct,
                          zero_copy_pct_wide=zc_pct_wide, type_v=w.type_v)
    h = kvs.kvs_create(cfg, local)
    rc = kvs.kvs_get_config(h)
    pb = kvs.kvs_page_bytes(rc)
    stream = torch.cuda.Stream(device=dev)

    # ---- history pre-fill (untimed) ----
    def prefill_history(hh):
        for layer in range(L):
            pos = 0
            while pos < w.pos0:
                n = min(16384, w.pos0 - pos)
                k, v = W.kv_tokens(w, layer, pos, pos + n)
                kd = torch.from_numpy(k).to(dev)
                vd = torch.from_numpy(v).to(dev)
                with torch.cuda.stream(stream):
                    kvs.kvs_append(hh, layer, pos, n, kd, vd, stream)
                stream.synchronize()
                pos += n

    t0 = time.time()
    prefill_history(h)
    prefill_s = time.time() - t0

    # ---- per-step inputs resident in HBM ----
    ks, vs, qs = [], [], []
    for layer in range(L):
        k, v = W.kv_tokens(w, layer, w.pos0, w.ctx)
        ks.append(torch.from_numpy(k).to(dev))
        vs.append(torch.from_numpy(v).to(dev))
        qs.append(torch.from_numpy(W.queries(w, layer, w.pos0)).to(dev))
    out = torch.empty((L, w.n_q, w.n_q_heads, 128), dtype=torch.float32, device=dev)
    lse = torch.empty((L, w.n_q, w.n_q_heads), dtype=torch.float32, device=dev)

    def one_step(k_in, v_in, q_in, o, l, hh=None):
        hh = h if hh is None else hh
        for layer in range(L):
            kvs.kvs_append(hh, layer, w.pos0, w.n_q, k_in[layer], v_in[layer], stream)
            kvs.kvs_attend(hh, layer, w.pos0, w.n_q, q_in[layer], o[layer], l[layer], stream)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dist if world > 1 else None, dev)

    for _ in range(args.warmup):
        one_step(ks, vs, qs, out, lse)
    barrier()
    h2d_before = best_big_copy_gbs(torch, dev)
    kvs.kvs_reset_stats(h)
    one_step(ks, vs, qs, out, lse)
    barrier()
    launches_per_step = int(kvs.kvs_get_stats(h)["kernel_launches"])

    # The timed steps are replays of one step (append + attend of every layer)
    # captured into a CUDA graph: the library's copy stream and side streams
    # join the capture.  The same steps issued as plain library calls are
    # timed afterwards and reported beside them ("eager").
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            one_step(ks, vs, qs, out, lse)
        for _ in range(args.warmup):
            with torch.cuda.stream(stream):
                graph.replay()
        barrier()

    def timed_step():
        if graph is not None:
            with torch.cuda.stream(stream):
                graph.replay()
        else:
            one_step(ks, vs, qs, out, lse)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.25)
    barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev[0].record(stream)
    for i in range(args.steps):
        timed_step()
        ev[i + 1].record(stream)
    barrier()
    ms_total = max_over_ranks(ev[0].elapsed_time(ev[-1]))
    ms_median = statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps))
    clk = clocks.stop()
    # library kernels launched in the timed region: a replay launches what one
    # plain step launched (counted above)
    gpu_launches = launches_per_step * args.steps
    ms_step = ms_total / args.steps
    value = job_value(world, w.ctx, L, ms_step)
    e0, e1 = ev[0], ev[-1]
    if graph is not None:
        del graph
        barrier()

    # the same steps as plain library calls issued by the host without waiting
    eager_line = None
    if args.graph:
        kvs.kvs_reset_stats(h)
        e0.record(stream)
        for _ in range(args.steps):
            one_step(ks, vs, qs, out, lse)
        e1.record(stream)
        barrier()
        ms_eager = max_over_ranks(e0.elapsed_time(e1)) / args.steps
        eager_line = {"ms_per_step": ms_eager, "value": job_value(world, w.ctx, L, ms_eager),
                      "unit": UNIT, "kernel_launches": int(kvs.kvs_get_stats(h)["kernel_launches"])}

    # ---- comparison arms: the same steps with the streamed pages split
    #      differently between the copy-engine ring and in-place reads of the
    #      mapped pinned history by the decode kernel (the share is switched
    #      on the same handle: its partial buffer is sized for every share) ----
    arms = {}
    if args.arms and zc_able:
        for name, pct in (("ring_only", 0), ("zero_copy_only", 100)):
            if pct == zc_pct:
                continue
            kvs.kvs_set_zero_copy_pct(h, -1 if wide else pct, pct if wide else -1)
            for _ in range(args.warmup):
                one_step(ks, vs, qs, out, lse)
            barrier()
            e0.record(stream)
            for _ in range(args.steps):
                one_step(ks, vs, qs, out, lse)
            e1.record(stream)
            barrier()
            ms_a = max_over_ranks(e0.elapsed_time(e1)) / args.steps
            S_a = w.n_pages - rc.n_resident_pages
            arms[name] = {"zero_copy_pct": pct, "ms_per_step": ms_a,
                          "value": job_value(world, w.ctx, L, ms_a), "unit": UNIT,
                          "h2d_gbs_achieved": L * S_a * pb / (ms_a * 1e-3) / 1e9,
                          "launch": "plain library calls"}
        kvs.kvs_set_zero_copy_pct(h, 0 if wide else zc_pct, zc_pct_wide)

    # ---- end to end through the C ABI with pinned host buffers ----
    kh = [x.cpu().pin_memory() for x in ks]
    vh = [x.cpu().pin_memory() for x in vs]
    qh = [x.cpu().pin_memory() for x in qs]
    oh = torch.empty(tuple(out.shape), dtype=torch.float32).pin_memory()
    lh = torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory()
    for _ in range(max(1, args.warmup // 2)):
        one_step(kh, vh, qh, oh, lh)
    barrier()
    e0.record(stream)
    e2e_steps = max(1, args.steps // 2)
    for _ in range(e2e_steps):
        one_step(kh, vh, qh, oh, lh)
    e1.record(stream)
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1)) / e2e_steps
    h2d_b = sum(x.numel() * x.element_size() for x in kh + vh + qh)
    d2h_b = oh.numel() * 4 + lh.numel() * 4

    # ---- kernel timing: the same steps again, with CUDA events around every
    #      launch of the library's kernels (a separate timed pass, so the
    #      events' host cost does not enter the step time above) ----
    st_prof = None
    if args.profile:
        kvs.kvs_set_profiling(h, True)
        one_step(ks, vs, qs, out, lse)
        barrier()
        kvs.kvs_reset_stats(h)
        for _ in range(min(args.steps, 60)):
            one_step(ks, vs, qs, out, lse)
        barrier()
        st_prof = kvs.kvs_get_stats(h)
        kvs.kvs_set_profiling(h, False)

    # ---- copy bandwidth of this machine (roofline denominator) ----
    chunk_b = rc.chunk_pages * pb if rc.chunk_pages else pb
    h2d_ring = kvs.kvs_measure_h2d(h, chunk_b, min(1 << 30, L * rc.n_resident_pages * pb), 10) \
        if rc.n_ring_slots else None
    # the best 64 MiB-copy rate, measured before the timed region and again
    # now (the larger is kept: a link shared with other work on the host can
    # read low in one of them, which would flatter every fraction)
    h2d_peak = max(h2d_before, best_big_copy_gbs(torch, dev), h2d_ring or 0.0)

    # ---- copy / compute timeline of a few plain steps, at the tuned share and
    #      ring-only (optional: --timeline DIR) ----
    timeline = None
    if args.timeline and rank == 0:
        os.makedirs(args.timeline, exist_ok=True)
        timeline = {}
        shares = [("tuned", zc_pct)] + ([("ring_only", 0)] if zc_able and zc_pct != 0 else [])
        for tag, pct in shares:
            kvs.kvs_set_zero_copy_pct(h, -1 if wide else pct, pct if wide else -1)
            for _ in range(2):
                one_step(ks, vs, qs, out, lse)
            path = os.path.join(args.timeline, f"timeline_{w.name}_{tag}.json")
            n_tl = 3
            capture_timeline(lambda: one_step(ks, vs, qs, out, lse), n_tl, path, barrier)
            timeline[tag] = timeline_summary(path, n_tl, h2d_peak)
            if timeline[tag] is not None:
                timeline[tag]["zero_copy_pct"] = pct
        kvs.kvs_set_zero_copy_pct(h, 0 if wide else zc_pct, zc_pct_wide)
        if args.graph:
            # replays of one captured step at the tuned share: consecutive
            # replays cannot overlap, so each boundary shows its tail
            g_tl = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_tl, stream=stream):
                one_step(ks, vs, qs, out, lse)

            def replay():
                with torch.cuda.stream(stream):
                    g_tl.replay()

            for _ in range(2):
                replay()
            path = os.path.join(args.timeline, f"timeline_{w.name}_tuned_graph.json")
            n_tl = 4
            capture_timeline(replay, n_tl, path, barrier)
            timeline["tuned_graph"] = timeline_summary(path, n_tl, h2d_peak)
            del g_tl
            barrier()

    hbm_peak, peak_src = peaks()
    P = w.n_pages
    R = min(rc.n_resident_pages, P)
    S = P - R
    t_roof = L * max(R * pb / (hbm_peak * 1e9), S * pb / (h2d_peak * 1e9))
    roof_frac = t_roof / (ms_step * 1e-3)
    # the same bound with the copy bandwidth of ring-sized chunks (the most a
    # ring of this many slots can be fed at), and the HBM term that also counts
    # the ring's own write and read of every streamed page
    t_roof_chunk = L * max(R * pb / (hbm_peak * 1e9), S * pb / (h2d_ring * 1e9)) if h2d_ring else t_roof
    t_hbm_ring = L * (R + 2 * S) * pb / (hbm_peak * 1e9)
    for arm in arms.values():
        arm["frac"] = t_roof / (arm["ms_per_step"] * 1e-3)
    vis_keys = sum(w.pos0 + j + 1 for j in range(w.n_q))
    step_flops = L * 4.0 * w.n_q_heads * 128 * vis_keys

    # Roofline of each kind of launch in the profiled pass, and of the dominant
    # one (largest summed launch time):
    #   decode_kernel (TMA): resident pages and ring slots, bound by HBM;
    #   decode_kernel (in place): streamed pages read over PCIe from the mapped
    #     pinned history, bound by the host-to-device link;
    #   chunk_mma_kernel: tensor cores.
    kernel = None
    kinds = {}
    if st_prof:
        prof_steps = min(args.steps, 60)
        ms_dec = st_prof["ms_decode_resident"] + st_prof["ms_decode_ring"]
        n_dec = st_prof["n_decode_resident"] + st_prof["n_decode_ring"]
        if n_dec > 0:
            bytes_k = st_prof["bytes_decode_resident"] + st_prof["bytes_decode_ring"]
            achieved = bytes_k / (ms_dec * 1e-3) / 1e9
            kinds["decode_kernel"] = (ms_dec, {
                "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak,
                "traffic": ncu_traffic("decode_kernel", w, pb, st_prof["bytes_decode_resident"],
                                       st_prof["bytes_decode_ring"], n_dec),
                "kernel": "decode_kernel", "launches": n_dec, "avg_launch_us": ms_dec / n_dec * 1e3,
                "bytes_per_launch": bytes_k / n_dec,
                "resident_only": {
                    "achieved": st_prof["bytes_decode_resident"] / max(st_prof["ms_decode_resident"], 1e-9) / 1e6,
                    "launches": st_prof["n_decode_resident"],
                    "avg_launch_us": st_prof["ms_decode_resident"] / max(1, st_prof["n_decode_resident"]) * 1e3}})
        ms_zc, n_zc = st_prof["ms_decode_zc"], st_prof["n_decode_zc"]

        def zc_traffic(kind):
            return ncu_in_place(w, pb, kind, st_prof["bytes_decode_zc"] / pb / n_zc)

        if n_zc > 0:
            achieved = st_prof["bytes_decode_zc"] / (ms_zc * 1e-3) / 1e9
            kinds["decode_kernel_in_place"] = (ms_zc, {
                "bound": "h2d", "bound_note": "the host-to-device PCIe link: the launch reads host memory",
                "achieved": achieved, "peak": h2d_peak, "unit": "GB/s",
                "frac": achieved / h2d_peak, "traffic": zc_traffic("dram"),
                "sysmem_traffic": zc_traffic("pcie"),
                "traffic_note": "traffic: DRAM bytes of a launch (Q and the split partials); "
                                "sysmem_traffic: host-memory bytes it reads over PCIe (ncu "
                                "pcie__read_bytes.sum per page of the capture x its pages)",
                "kernel": "decode_kernel (in-place reads of streamed pages)", "launches": n_zc,
                "avg_launch_us": ms_zc / n_zc * 1e3, "bytes_per_launch": st_prof["bytes_decode_zc"] / n_zc,
                "peak_note": "best pinned host-to-device copy rate measured in this run"})
        ms_tz, n_tz = st_prof["ms_chunk_zc"], st_prof["n_chunk_zc"]
        if n_tz > 0:
            achieved = st_prof["bytes_chunk_zc"] / (ms_tz * 1e-3) / 1e9
            kinds["chunk_mma_kernel_in_place"] = (ms_tz, {
                "bound": "h2d", "bound_note": "the host-to-device PCIe link: the launch reads host memory",
                "achieved": achieved, "peak": h2d_peak, "unit": "GB/s", "frac": achieved / h2d_peak,
                "traffic": None, "kernel": "chunk_mma_kernel (in-place reads of streamed pages)",
                "launches": n_tz, "avg_launch_us": ms_tz / n_tz * 1e3,
                "bytes_per_launch": st_prof["bytes_chunk_zc"] / n_tz,
                "peak_note": "best pinned host-to-device copy rate measured in this run"})
        ms_tc, n_tc = st_prof["ms_chunk_mma"], st_prof["n_chunk_mma"]
        if n_tc > 0:
            # algorithmic flops: QK^T and PV over every visible key of every query row
            vis = sum(w.pos0 + j + 1 for j in range(w.n_q))
            flops = prof_steps * L * 4.0 * w.n_q_heads * 128 * vis
            # the share of the keys these (TMA-fed) launches attend; the
            # in-place launches attend the rest
            S_ = w.n_pages - min(rc.n_resident_pages, w.n_pages)
            S_zc_ = min(S_, (S_ * zc_pct_wide + 50) // 100)
            flops *= (w.n_pages - S_zc_) / w.n_pages
            achieved = flops / (ms_tc * 1e-3) / 1e12
            tc_peak = peak_tflops()
            res_b = prof_steps * L * min(rc.n_resident_pages, w.n_pages) * pb
            ring_b = prof_steps * L * (S_ - S_zc_) * pb
            kinds["chunk_mma_kernel"] = (ms_tc, {
                "bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved / tc_peak,
                "traffic": ncu_traffic("chunk_mma_kernel", w, pb, res_b, ring_b, n_tc),
                "kernel": "chunk_mma_kernel", "launches": n_tc, "avg_launch_us": ms_tc / n_tc * 1e3,
                "flops_per_launch": flops / n_tc,
                "peak_note": "measured dense bf16 burst; fp16 has the same nominal rate"})
        if kinds:
            total = sum(ms for ms, _ in kinds.values())
            name = max(kinds, key=lambda k: kinds[k][0])
            kernel = dict(kinds[name][1])
            kernel.update({
                "peak_source": peak_src, "time_share": kinds[name][0] / total,
                "timing": "CUDA events around each launch on its stream; separate pass of the same "
                          "steps with the library's kernels serialized on one stream",
                "other_kinds": {k: {"frac": v[1]["frac"], "bound": v[1]["bound"], "time_share": v[0] / total,
                                    "avg_launch_us": v[1]["avg_launch_us"]}
                                for k, v in kinds.items() if k != name} or None,
                "other_kernels_avg_us": {
                    "merge": st_prof["ms_merge"] / max(1, st_prof["n_merge"]) * 1e3,
                    "append": st_prof["ms_append"] / max(1, st_prof["n_append"]) * 1e3}})

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16*f16->f32",  # tensor-core operands (exact codes), fp32 accumulate/softmax
        "data": "synthetic",
        "config": {"workload": w.name, "ctx": w.ctx, "n_layers": L, "n_q": w.n_q,
                   "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": 128,
                   "kv_types": "K q8_0 / V " + {8: "q8_0", 6: "q5_0", 3: "q4_1", 7: "q5_1"}.get(w.type_v, "q4_0"),
                   "page_tokens": 256, "resident_pages": R,
                   "streamed_pages": S, "ring_slots": rc.n_ring_slots, "chunk_pages": rc.chunk_pages,
                   "zero_copy_pct": zc_pct, "zero_copy_share_of": "tensor-core calls" if wide else "decode calls",
                   "parallelism": f"replicas{world}", "l2": "inputs larger than L2 (resident "
                   f"{L * R * pb / 1e6:.0f} MB + streamed {L * S * pb / 1e6:.0f} MB per step)",
                   },
        "roofline": kernel,
        "step_roofline": {"bound": "h2d" if S * pb / h2d_peak > R * pb / hbm_peak else "hbm",
                          "t_roof_ms": t_roof * 1e3, "t_step_ms": ms_step, "frac": roof_frac,
                          "h2d_gbs_peak_measured": h2d_peak, "h2d_gbs_ring_chunk": h2d_ring,
                          "h2d_gbs_achieved": L * S * pb / (ms_step * 1e-3) / 1e9,
                          "frac_at_ring_chunk_h2d": t_roof_chunk / (ms_step * 1e-3),
                          "hbm_ms_incl_ring_write_read": t_hbm_ring * 1e3,
                          "tensor_ms_at_peak": step_flops / (peak_tflops() * 1e12) * 1e3,
                          "step_flops": step_flops,
                          "hbm_gbs_peak": hbm_peak, "peak_source": peak_src},
        "e2e": {"value": world * w.ctx * L / (ms_e2e * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b, "ms_per_step": ms_e2e},
        "gpu_launches": gpu_launches,
        "launch": "replays of one captured step (CUDA graph)" if args.graph else "plain library calls",
        "eager": eager_line,
        "arms": arms or None,
        "ms_per_step_median": ms_median,
        "clocks": clk,
        "prefill_s": prefill_s,
    }
    if timeline is not None:
        line["timeline"] = timeline
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    del timed_step
    torch.cuda.synchronize(dev)
    kvs.kvs_destroy(h)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=W.DEFAULT_BENCH, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--chunk-pages", type=int, default=0)
    ap.add_argument("--no-profile", dest="profile", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-arms", dest="arms", action="store_false",
                    help="skip the ring-only / zero-copy-only comparison arms")
    ap.add_argument("--zero-copy-pct", type=int, default=-1,
                    help="share of streamed pages decode reads in place (default: the tuned share)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time plain library calls instead of replays of a captured step")
    ap.add_argument("--timeline", default="",
                    help="directory: after timing, record a few plain steps' copy/compute timeline "
                         "(Chrome trace) and add its summary to the line")
    args = ap.parse_args()
    w = W.WORKLOADS[args.workload]
    if args.steps <= 0:
        # a timed region of a few seconds
        args.steps = {"tiny_decode_4k": 2000, "streamed_decode_32k": 300, "streamed_decode_32k_q8v": 240,
                      "streamed_decode_32k_q5v": 280, "streamed_decode_32k_q41v": 280,
                      "streamed_decode_32k_q51v": 260,
                      "long_decode_256k": 30,
                      "verify_128k": 60, "prefill_chunk_64k": 200}[w.name]
        if args.impl == "reference":
            args.steps = 5
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
