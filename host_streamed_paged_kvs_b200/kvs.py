"""Thin Python binding of libkvs (include/kvs.h).

Argument marshalling only: every step of the path runs in the CUDA library.
Tensors are passed by address (torch CUDA tensors, pinned or plain CPU tensors,
numpy arrays); streams by their cudaStream_t handle.  There is no fallback:
importing this module fails loudly if libkvs.so has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvs.so")

KVS_OK = 0
KVS_E_INVAL = -1
KVS_E_ARENA = -2
KVS_E_WIDTH = -3
KVS_E_ORDER = -4
KVS_E_CUDA = -5
KVS_E_TIMEOUT = -6
KVS_E_NOMEM = -7
KVS_TYPE_F16 = 1
KVS_TYPE_Q4_0 = 2
KVS_TYPE_Q4_1 = 3
KVS_TYPE_Q5_0 = 6
KVS_TYPE_Q5_1 = 7
KVS_TYPE_Q8_0 = 8
KVS_PAGE_ABSENT = -1
KVS_PAGE_RESIDENT = 1
KVS_PAGE_STREAMED = 2
KVS_FLAG_PROFILE = 1
KVS_FLAG_PHASE_ARENA = 2
KVS_PHASE_PREFILL = 0
KVS_PHASE_DECODE = 1

ERROR_NAMES = {0: "KVS_OK", -1: "KVS_E_INVAL", -2: "KVS_E_ARENA", -3: "KVS_E_WIDTH",
               -4: "KVS_E_ORDER", -5: "KVS_E_CUDA", -6: "KVS_E_TIMEOUT", -7: "KVS_E_NOMEM"}

# every symbol the header declares
EXPORTS = ["kvs_resolve_config", "kvs_page_bytes", "kvs_plan_page", "kvs_plan_ring", "kvs_create", "kvs_destroy",
           "kvs_append", "kvs_attend", "kvs_export_page", "kvs_page_location", "kvs_layer_length",
           "kvs_get_config", "kvs_get_stats", "kvs_reset_stats", "kvs_set_profiling",
           "kvs_set_zero_copy_pct", "kvs_sync",
           "kvs_measure_h2d", "kvs_attend_pages_static", "kvs_selftest_bounded_wait",
           "kvs_last_error", "kvs_eject_init", "kvs_eject_step", "kvs_draft_capacity_pages",
           "kvs_phase_layout", "kvs_set_phase", "kvs_pin", "kvs_draft_eject", "kvs_draft_restore",
           "kvs_get_arena"]


class kvs_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("page_tokens", ctypes.c_int), ("max_ctx", ctypes.c_int),
                ("n_resident_pages", ctypes.c_int), ("n_ring_slots", ctypes.c_int),
                ("max_q_tokens", ctypes.c_int), ("type_k", ctypes.c_int),
                ("type_v", ctypes.c_int), ("chunk_pages", ctypes.c_int),
                ("flags", ctypes.c_int), ("zero_copy_pct", ctypes.c_int),
                ("arena_bytes", ctypes.c_size_t), ("n_aux_layers", ctypes.c_int),
                ("aux_resident_pages", ctypes.c_int), ("zero_copy_pct_wide", ctypes.c_int)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class kvs_arena_status(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int) for n in ("phase", "width", "n_resident_pages", "aux_resident_pages",
                                             "draft_active", "phase_arena")] +
                [(n, ctypes.c_size_t) for n in ("arena_bytes", "compute_bytes", "resident_bytes", "ring_bytes",
                                                "aux_bytes", "pinned_bytes", "free_bytes")])

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class kvs_stats(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_uint64) for n in
                 ("appends", "attends", "tokens_appended", "pages_streamed", "bytes_h2d",
                  "bytes_resident_read", "h2d_copies", "kernel_launches")] +
                [(n, ctypes.c_double) for n in
                 ("ms_decode_resident", "ms_decode_ring", "ms_merge", "ms_append", "ms_chunk_mma",
                  "ms_decode_zc")] +
                [(n, ctypes.c_uint64) for n in
                 ("n_decode_resident", "n_decode_ring", "n_merge", "n_append", "n_chunk_mma",
                  "n_decode_zc", "bytes_decode_resident", "bytes_decode_ring", "bytes_decode_zc")] +
                [("ms_chunk_zc", ctypes.c_double), ("n_chunk_zc", ctypes.c_uint64),
                 ("bytes_chunk_zc", ctypes.c_uint64)])

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class kvs_eject_params(ctypes.Structure):
    _fields_ = [("keep_pages", ctypes.c_int), ("reenable_pages", ctypes.c_int),
                ("stable_decodes", ctypes.c_int), ("capacity_pages", ctypes.c_int)]


class kvs_eject_state(ctypes.Structure):
    _fields_ = [("draft_active", ctypes.c_int), ("streak", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libkvs.so not found at {LIB_PATH}: build it with "
            "`python -m host_streamed_paged_kvs_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, cp = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER
    L.kvs_resolve_config.argtypes = [cp(kvs_config), cp(kvs_config), cp(ctypes.c_size_t)]
    L.kvs_page_bytes.restype = ctypes.c_size_t
    L.kvs_page_bytes.argtypes = [cp(kvs_config)]
    L.kvs_plan_page.argtypes = [cp(kvs_config), i, i, cp(i), cp(i)]
    L.kvs_plan_ring.argtypes = [cp(kvs_config), i, i, ctypes.c_longlong, cp(i), cp(i), cp(i), i]
    L.kvs_create.argtypes = [cp(kvs_config), i, cp(vp)]
    L.kvs_destroy.argtypes = [vp]
    L.kvs_destroy.restype = None
    L.kvs_append.argtypes = [vp, i, i, i, vp, vp, vp]
    L.kvs_attend.argtypes = [vp, i, i, i, vp, vp, vp, vp]
    L.kvs_export_page.argtypes = [vp, i, i, i, vp]
    L.kvs_page_location.argtypes = [vp, i, i, cp(i), cp(i)]
    L.kvs_layer_length.argtypes = [vp, i, cp(i)]
    L.kvs_get_config.argtypes = [vp, cp(kvs_config)]
    L.kvs_get_stats.argtypes = [vp, cp(kvs_stats)]
    L.kvs_reset_stats.argtypes = [vp]
    L.kvs_set_profiling.argtypes = [vp, i]
    L.kvs_set_zero_copy_pct.argtypes = [vp, i, i]
    L.kvs_sync.argtypes = [vp, vp, ctypes.c_double]
    L.kvs_measure_h2d.argtypes = [vp, ctypes.c_size_t, ctypes.c_size_t, i, cp(ctypes.c_double)]
    L.kvs_attend_pages_static.argtypes = [vp, i, i, i, i, i, i, vp, vp, vp, vp]
    L.kvs_selftest_bounded_wait.argtypes = [i, ctypes.c_double, cp(i)]
    L.kvs_last_error.restype = ctypes.c_char_p
    L.kvs_last_error.argtypes = [vp]
    L.kvs_eject_init.argtypes = [cp(kvs_eject_params), cp(kvs_eject_state)]
    L.kvs_eject_step.argtypes = [cp(kvs_eject_params), cp(kvs_eject_state), i]
    L.kvs_draft_capacity_pages.argtypes = [cp(kvs_config), ctypes.c_size_t, cp(i)]
    L.kvs_phase_layout.argtypes = [cp(kvs_config), i, ctypes.c_size_t, i, cp(kvs_arena_status)]
    L.kvs_set_phase.argtypes = [vp, i, i, vp]
    L.kvs_pin.argtypes = [vp, ctypes.c_size_t, cp(vp), vp]
    L.kvs_draft_eject.argtypes = [vp, vp]
    L.kvs_draft_restore.argtypes = [vp, vp]
    L.kvs_get_arena.argtypes = [vp, cp(kvs_arena_status)]
    return L


lib = _load()


class KvsError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def _addr(x) -> Optional[int]:
    """Address of a tensor / array / raw int (None -> NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream  # torch.cuda.Stream


def _check(rc: int, handle=None):
    if rc != KVS_OK:
        raise KvsError(rc, lib.kvs_last_error(handle).decode())


def make_config(n_layers, n_q_heads, n_kv_heads, max_ctx, n_resident_pages=0, n_ring_slots=0,
                max_q_tokens=1, chunk_pages=0, flags=0, arena_bytes=0, head_dim=128,
                page_tokens=256, type_k=KVS_TYPE_Q8_0, type_v=KVS_TYPE_Q4_0,
                zero_copy_pct=0, n_aux_layers=0, aux_resident_pages=0,
                zero_copy_pct_wide=0) -> kvs_config:
    return kvs_config(n_layers, n_q_heads, n_kv_heads, head_dim, page_tokens, max_ctx,
                      n_resident_pages, n_ring_slots, max_q_tokens, type_k, type_v, chunk_pages,
                      flags, zero_copy_pct, arena_bytes, n_aux_layers, aux_resident_pages,
                      zero_copy_pct_wide)


# ---- functions with the C names ------------------------------------------

def kvs_resolve_config(cfg: kvs_config):
    out = kvs_config()
    hb = ctypes.c_size_t()
    _check(lib.kvs_resolve_config(ctypes.byref(cfg), ctypes.byref(out), ctypes.byref(hb)))
    return out, hb.value


def kvs_page_bytes(cfg: kvs_config) -> int:
    return lib.kvs_page_bytes(ctypes.byref(cfg))


def kvs_plan_page(cfg: kvs_config, n_tokens: int, page: int):
    k, i = ctypes.c_int(), ctypes.c_int()
    _check(lib.kvs_plan_page(ctypes.byref(cfg), n_tokens, page, ctypes.byref(k), ctypes.byref(i)))
    return k.value, i.value


def kvs_plan_ring(cfg: kvs_config, n_q: int, s_ring: int, ring_ctr0: int = 0):
    """The ring schedule of one attend call: [(page0, pages, slot0), ...]."""
    n = lib.kvs_plan_ring(ctypes.byref(cfg), n_q, s_ring, ring_ctr0, None, None, None, 0)
    _check(n if n < 0 else 0)
    p0, pg, sl = (ctypes.c_int * max(1, n))(), (ctypes.c_int * max(1, n))(), (ctypes.c_int * max(1, n))()
    _check(min(0, lib.kvs_plan_ring(ctypes.byref(cfg), n_q, s_ring, ring_ctr0, p0, pg, sl, n)))
    return [(p0[k], pg[k], sl[k]) for k in range(n)]


def kvs_create(cfg: kvs_config, device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(lib.kvs_create(ctypes.byref(cfg), device, ctypes.byref(h)))
    return h.value


def kvs_destroy(h: int) -> None:
    lib.kvs_destroy(h)


def kvs_append(h, layer, pos0, n_tok, k, v, stream=None) -> None:
    _check(lib.kvs_append(h, layer, pos0, n_tok, _addr(k), _addr(v), _stream(stream)), h)


def kvs_attend(h, layer, pos0, n_q, q, out, lse=None, stream=None) -> None:
    _check(lib.kvs_attend(h, layer, pos0, n_q, _addr(q), _addr(out), _addr(lse), _stream(stream)), h)


def kvs_export_page(h, layer, page, from_device, dst) -> None:
    _check(lib.kvs_export_page(h, layer, page, int(from_device), _addr(dst)), h)


def kvs_page_location(h, layer, page):
    k, i = ctypes.c_int(), ctypes.c_int()
    _check(lib.kvs_page_location(h, layer, page, ctypes.byref(k), ctypes.byref(i)), h)
    return k.value, i.value


def kvs_layer_length(h, layer) -> int:
    n = ctypes.c_int()
    _check(lib.kvs_layer_length(h, layer, ctypes.byref(n)), h)
    return n.value


def kvs_get_config(h) -> kvs_config:
    c = kvs_config()
    _check(lib.kvs_get_config(h, ctypes.byref(c)), h)
    return c


def kvs_get_stats(h) -> dict:
    s = kvs_stats()
    _check(lib.kvs_get_stats(h, ctypes.byref(s)), h)
    return s.as_dict()


def kvs_reset_stats(h) -> None:
    _check(lib.kvs_reset_stats(h), h)


def kvs_set_profiling(h, enable: bool) -> None:
    _check(lib.kvs_set_profiling(h, int(bool(enable))), h)


def kvs_set_zero_copy_pct(h, pct: int = -1, pct_wide: int = -1) -> None:
    """In-place shares for decode calls and wider calls; -1 leaves one unchanged."""
    _check(lib.kvs_set_zero_copy_pct(h, int(pct), int(pct_wide)), h)


def kvs_phase_layout(cfg: kvs_config, width: int, pinned_bytes: int = 0, draft_active: bool = True) -> dict:
    st = kvs_arena_status()
    _check(lib.kvs_phase_layout(ctypes.byref(cfg), int(width), int(pinned_bytes), int(bool(draft_active)),
                                ctypes.byref(st)))
    return st.as_dict()


def kvs_set_phase(h, phase: int, width: int = 0, stream=None) -> None:
    _check(lib.kvs_set_phase(h, int(phase), int(width), _stream(stream)), h)


def kvs_pin(h, nbytes: int, stream=None) -> int:
    p = ctypes.c_void_p()
    _check(lib.kvs_pin(h, int(nbytes), ctypes.byref(p), _stream(stream)), h)
    return p.value


def kvs_draft_eject(h, stream=None) -> None:
    _check(lib.kvs_draft_eject(h, _stream(stream)), h)


def kvs_draft_restore(h, stream=None) -> None:
    _check(lib.kvs_draft_restore(h, _stream(stream)), h)


def kvs_get_arena(h) -> dict:
    st = kvs_arena_status()
    _check(lib.kvs_get_arena(h, ctypes.byref(st)), h)
    return st.as_dict()


def kvs_sync(h, stream=None, timeout_s: float = 60.0) -> None:
    _check(lib.kvs_sync(h, _stream(stream), timeout_s), h)


def kvs_measure_h2d(h, chunk_bytes: int, total_bytes: int, reps: int = 10) -> float:
    g = ctypes.c_double()
    _check(lib.kvs_measure_h2d(h, chunk_bytes, total_bytes, reps, ctypes.byref(g)), h)
    return g.value


def kvs_attend_pages_static(pages, n_pages, n_tokens, n_q_heads, n_kv_heads, pos0, n_q, q, out,
                            lse=None, stream=None) -> None:
    """No-allocation attention over caller-owned device pages (see include/kvs.h)."""
    _check(lib.kvs_attend_pages_static(_addr(pages), n_pages, n_tokens, n_q_heads, n_kv_heads, pos0,
                                       n_q, _addr(q), _addr(out), _addr(lse), _stream(stream)))


KVS_ERR_WAIT_TIMEOUT = 1


def kvs_selftest_bounded_wait(device: int = 0, limit_s: float = 0.2) -> int:
    bits = ctypes.c_int()
    _check(lib.kvs_selftest_bounded_wait(device, limit_s, ctypes.byref(bits)))
    return bits.value


def kvs_last_error(h=None) -> str:
    return lib.kvs_last_error(h).decode()


def kvs_eject_init(keep_pages=0, reenable_pages=0, stable_decodes=0, capacity_pages=0):
    """Returns (params with defaults filled, state with the draft active)."""
    p = kvs_eject_params(keep_pages, reenable_pages, stable_decodes, capacity_pages)
    s = kvs_eject_state()
    _check(lib.kvs_eject_init(ctypes.byref(p), ctypes.byref(s)))
    return p, s


def kvs_eject_step(params: kvs_eject_params, state: kvs_eject_state, working_pages: int) -> bool:
    """One decode batch; True when the draft was ejected or re-enabled."""
    rc = lib.kvs_eject_step(ctypes.byref(params), ctypes.byref(state), int(working_pages))
    _check(rc if rc < 0 else 0)
    return rc == 1


def kvs_draft_capacity_pages(cfg: kvs_config, pinned_bytes: int) -> int:
    n = ctypes.c_int()
    _check(lib.kvs_draft_capacity_pages(ctypes.byref(cfg), int(pinned_bytes), ctypes.byref(n)))
    return n.value


class KVS:
    """Owning handle with the same calls as methods."""

    def __init__(self, cfg: kvs_config, device: int = 0):
        self.h = kvs_create(cfg, device)
        self.cfg = kvs_get_config(self.h)

    def append(self, layer, pos0, n_tok, k, v, stream=None):
        kvs_append(self.h, layer, pos0, n_tok, k, v, stream)

    def attend(self, layer, pos0, n_q, q, out, lse=None, stream=None):
        kvs_attend(self.h, layer, pos0, n_q, q, out, lse, stream)

    def export_page(self, layer, page, from_device, dst):
        kvs_export_page(self.h, layer, page, from_device, dst)

    def page_location(self, layer, page):
        return kvs_page_location(self.h, layer, page)

    def layer_length(self, layer):
        return kvs_layer_length(self.h, layer)

    def stats(self):
        return kvs_get_stats(self.h)

    def reset_stats(self):
        kvs_reset_stats(self.h)

    def sync(self, stream=None, timeout_s=60.0):
        kvs_sync(self.h, stream, timeout_s)

    def measure_h2d(self, chunk_bytes, total_bytes, reps=10):
        return kvs_measure_h2d(self.h, chunk_bytes, total_bytes, reps)

    def close(self):
        if self.h:
            kvs_destroy(self.h)
            self.h = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
