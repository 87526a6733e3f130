"""ctypes binding of libmoe (include/moe.h): the same names, argument
marshalling only.  Device buffers are torch CUDA tensors (or raw device
addresses); every step of the path runs in the library's CUDA kernels.

The library is loaded from this package directory.  If it is missing the
first call raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID, MOE_ERR_CUDA, MOE_ERR_UNSUPPORTED, MOE_ERR_NOT_RESIDENT, MOE_ERR_CAPACITY, \
    MOE_ERR_TIMEOUT = range(7)
DEV_ERR_NOT_RESIDENT, DEV_ERR_SLOT_RANGE, DEV_ERR_TIMEOUT, DEV_ERR_BAD_EXPERT = 1, 2, 4, 8
WS_CONTROL_BYTES = 512  # head of the workspace: the control block (include/moe.h, moe_workspace_bytes)

# every entry point declared in include/moe.h
ABI_SYMBOLS = [
    "moe_slot_bytes", "moe_slot_layout", "moe_workspace_bytes", "moe_route", "moe_sort", "moe_slot_lookup",
    "moe_install_slots", "moe_expert_ffn", "moe_dequant_slot", "moe_quantize_rows", "moe_exp_portable",
    "moe_status_string", "moe_cache_create", "moe_cache_destroy", "moe_cache_table", "moe_cache_layer_base",
    "moe_cache_class_slots", "moe_cache_place", "moe_cache_step", "moe_cache_stats",
    "moe_expert_ffn_noalloc", "moe_noalloc_scratch_bytes", "moe_cache_resident", "moe_decode_layer",
    "moe_last_cuda_error", "moe_ffn_kernel_path", "moe_set_wait_limit_cycles", "moe_route_shared",
    "moe_router_logits", "moe_cache_reserve", "moe_cache_commit", "moe_prefetch_create", "moe_prefetch_destroy",
    "moe_prefetch_stats", "moe_decode_layer_ahead", "moe_route_sort_lookup", "moe_route_expert_ffn",
]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        extra = f" [{lib().moe_last_cuda_error().decode()}]" if status == MOE_ERR_CUDA else ""
        super().__init__(f"{where}: {status_string(status)} (status {status}){extra}")
        self.status = status


class LayerDesc(C.Structure):
    _fields_ = [("E", C.c_int32), ("k", C.c_int32), ("H", C.c_int32), ("I", C.c_int32), ("group", C.c_int32),
                ("bits_gu", C.c_int32), ("bits_down", C.c_int32)]

    def __repr__(self):
        return (f"LayerDesc(E={self.E}, k={self.k}, H={self.H}, I={self.I}, group={self.group}, "
                f"bits_gu={self.bits_gu}, bits_down={self.bits_down})")


class StepBuffers(C.Structure):
    _fields_ = [("ids", C.c_void_p), ("w", C.c_void_p), ("offsets", C.c_void_p), ("pairs", C.c_void_p),
                ("meta", C.c_void_p), ("meta_host", C.c_void_p), ("slots", C.c_void_p), ("dev_err", C.c_void_p),
                ("ws", C.c_void_p), ("ws_bytes", C.c_size_t), ("max_tokens", C.c_int32),
                ("x_sorted", C.c_void_p)]


class LayerCtx(C.Structure):
    _fields_ = [("desc", C.POINTER(LayerDesc)), ("pool", C.c_void_p), ("n_slots", C.c_int32),
                ("slot_bytes", C.c_size_t), ("table_dev", C.c_void_p), ("table_stage", C.c_void_p),
                ("bank_rows", C.POINTER(C.c_void_p)), ("n_shared", C.c_int32), ("shared_w", C.c_void_p)]


class Guess(C.Structure):
    _fields_ = [("layer", C.c_int32), ("lc", C.POINTER(LayerCtx)), ("logits", C.c_void_p), ("top", C.c_int32)]


class GuessBuffers(C.Structure):
    _fields_ = [("ids", C.c_void_p), ("w", C.c_void_p), ("ids_host", C.c_void_p), ("stride", C.c_int32)]


class SlotLayout(C.Structure):
    _fields_ = [("gate_up", C.c_uint64), ("down", C.c_uint64), ("gate_up_tile_bytes", C.c_uint64),
                ("down_tile_bytes", C.c_uint64), ("slot_bytes", C.c_uint64)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not built ({LIB_PATH}); run streamed_quantized_expert_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        P, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
        D = C.POINTER(LayerDesc)
        sig = {
            "moe_slot_bytes": (sz, [D]),
            "moe_slot_layout": (C.c_int, [D, C.POINTER(SlotLayout)]),
            "moe_workspace_bytes": (sz, [D, i32]),
            "moe_route": (C.c_int, [P, i32, D, f32, P, P, P, P]),
            "moe_route_shared": (C.c_int, [P, i32, D, f32, P, i32, P, P, P, P]),
            "moe_sort": (C.c_int, [P, P, i32, D, P, P, P, P, P, P, sz, P]),
            "moe_slot_lookup": (C.c_int, [P, P, P, i32, i32, i32, P, P, P, P, P]),
            "moe_route_sort_lookup": (C.c_int, [P, i32, D, f32, P, i32, P, i32, P, P, P, P, P, P, P, P, P, P, P]),
            "moe_route_expert_ffn": (C.c_int, [P, P, i32, D, f32, P, i32, P, P, P, P, P, P, P, P, P, P, P, P, sz, P,
                                               P]),
            "moe_install_slots": (C.c_int, [P, sz, i32, P, P, i32, P, P]),
            "moe_expert_ffn": (C.c_int, [P, i32, D, P, i32, P, P, P, P, P, P, P, P, i32, i32, P, P, sz, P, P]),
            "moe_expert_ffn_noalloc": (C.c_int, [P, i32, D, P, i32, P, P, P, P, P, P, P, i32, i32, P, P, P]),
            "moe_noalloc_scratch_bytes": (sz, []),
            "moe_dequant_slot": (C.c_int, [P, i32, D, P, P, P]),
            "moe_quantize_rows": (C.c_int, [P, i32, i32, i32, i32, i32, P, P]),
            "moe_exp_portable": (C.c_int, [P, i64, P, P]),
            "moe_status_string": (C.c_char_p, [C.c_int]),
            "moe_last_cuda_error": (C.c_char_p, []),
            "moe_ffn_kernel_path": (i32, [D, i32, i32]),
            "moe_set_wait_limit_cycles": (None, [i64]),
            "moe_cache_create": (C.c_int, [i32, i32, P, i32, C.POINTER(P)]),
            "moe_cache_destroy": (None, [P]),
            "moe_cache_table": (C.POINTER(i32), [P, i32]),
            "moe_cache_layer_base": (i32, [P, i32]),
            "moe_cache_class_slots": (i32, [P, i32]),
            "moe_cache_place": (C.c_int, [P, i32, P, P, i32]),
            "moe_cache_step": (C.c_int, [P, i32, P, i32, P, P, P]),
            "moe_cache_stats": (None, [P, P, P, P]),
            "moe_cache_resident": (i32, [P, i32]),
            "moe_decode_layer": (C.c_int, [P, i32, C.POINTER(LayerCtx), C.POINTER(StepBuffers), P, P, i32, f32, P,
                                           P, P, P, C.POINTER(i32)]),
            "moe_router_logits": (C.c_int, [P, i32, P, P, f32, i32, i32, P, P]),
            "moe_cache_reserve": (C.c_int, [P, i32, P, i32, P, P, P]),
            "moe_cache_commit": (C.c_int, [P, i32, i32, P]),
            "moe_prefetch_create": (C.c_int, [i32, C.POINTER(P)]),
            "moe_prefetch_destroy": (None, [P]),
            "moe_prefetch_stats": (None, [P, P, P, P, P, P]),
            "moe_decode_layer_ahead": (C.c_int, [P, P, i32, C.POINTER(LayerCtx), C.POINTER(StepBuffers), P, P, i32,
                                                 f32, P, P, P, P, C.POINTER(i32), C.POINTER(Guess), i32,
                                                 C.POINTER(GuessBuffers), P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


MOE_PATH_FUSED_DECODE, MOE_PATH_GEMV, MOE_PATH_TC_PREFILL = 0, 1, 2


def moe_ffn_kernel_path(d: LayerDesc, T: int, has_x_sorted: bool) -> int:
    """Kernels moe_expert_ffn runs for this layer shape and token count."""
    return int(lib().moe_ffn_kernel_path(C.byref(d), int(T), 1 if has_x_sorted else 0))


def moe_set_wait_limit_cycles(cycles: int) -> None:
    """Clock-cycle limit of every bounded device wait in kernels launched
    from now on (process-wide); 0 restores the default (4e9 cycles)."""
    lib().moe_set_wait_limit_cycles(int(cycles))


def status_string(s: int) -> str:
    return lib().moe_status_string(int(s)).decode()


def _ck(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t) -> int | None:
    """Device (or host) address of a tensor / int / None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream  # torch.cuda.Stream


def desc(E, k, H, I, group, bits_gu, bits_down=None) -> LayerDesc:
    return LayerDesc(E, k, H, I, group, bits_gu, bits_gu if bits_down is None else bits_down)


# ---------------------------------------------------------------------------
# sizes
# ---------------------------------------------------------------------------
def moe_slot_bytes(d: LayerDesc) -> int:
    return int(lib().moe_slot_bytes(C.byref(d)))


def moe_slot_layout(d: LayerDesc) -> SlotLayout:
    out = SlotLayout()
    _ck(lib().moe_slot_layout(C.byref(d), C.byref(out)), "moe_slot_layout")
    return out


def moe_workspace_bytes(d: LayerDesc, max_tokens: int) -> int:
    return int(lib().moe_workspace_bytes(C.byref(d), int(max_tokens)))


# ---------------------------------------------------------------------------
# stages
# ---------------------------------------------------------------------------
def moe_route(logits, T, d, L, slot_table, ids, w, stream=None) -> None:
    _ck(lib().moe_route(_ptr(logits), int(T), C.byref(d), float(L), _ptr(slot_table), _ptr(ids), _ptr(w),
                        _stream(stream)), "moe_route")


def moe_route_shared(logits, T, d, L, slot_table, n_shared, shared_w, ids, w, stream=None) -> None:
    _ck(lib().moe_route_shared(_ptr(logits), int(T), C.byref(d), float(L), _ptr(slot_table), int(n_shared),
                               _ptr(shared_w), _ptr(ids), _ptr(w), _stream(stream)), "moe_route_shared")


def widened(d: LayerDesc, n_shared: int) -> LayerDesc:
    """The description the calls after moe_route_shared take: E + n_shared
    experts, k + n_shared per token."""
    return desc(d.E + n_shared, d.k + n_shared, d.H, d.I, d.group, d.bits_gu, d.bits_down)


def moe_sort(ids, x, T, d, offsets, pairs, active, n_active, x_sorted, ws, ws_bytes, stream=None) -> None:
    _ck(lib().moe_sort(_ptr(ids), _ptr(x), int(T), C.byref(d), _ptr(offsets), _ptr(pairs), _ptr(active),
                       _ptr(n_active), _ptr(x_sorted), _ptr(ws), int(ws_bytes), _stream(stream)), "moe_sort")


def moe_route_sort_lookup(logits, T, d, L, slot_table, n_slots, ids, w, offsets, pairs, active, n_active, slots,
                          miss, n_miss, dev_err, stream=None, n_shared=0, shared_w=None) -> None:
    """moe_route_shared (moe_route when n_shared is 0) + moe_sort (no
    x_sorted) + moe_slot_lookup over the whole active list for one token, in
    one launch (T must be 1; d the routed experts' description)."""
    _ck(lib().moe_route_sort_lookup(_ptr(logits), int(T), C.byref(d), float(L), _ptr(slot_table), int(n_shared),
                                    _ptr(shared_w), int(n_slots), _ptr(ids), _ptr(w), _ptr(offsets), _ptr(pairs),
                                    _ptr(active), _ptr(n_active), _ptr(slots), _ptr(miss), _ptr(n_miss),
                                    _ptr(dev_err), _stream(stream)),
        "moe_route_sort_lookup")


def moe_route_expert_ffn(x, logits, T, d, L, pool, n_slots, slot_table, ids, w, offsets, pairs, active, n_active,
                         slots, miss, n_miss, y, ws, ws_bytes, dev_err, stream=None) -> None:
    """Routing, sort, lookup and FFN of one token of a resident layer in one
    launch (T must be 1): the stage outputs as moe_route_sort_lookup writes
    them, and y (overwritten)."""
    _ck(lib().moe_route_expert_ffn(_ptr(x), _ptr(logits), int(T), C.byref(d), float(L), _ptr(pool), int(n_slots),
                                   _ptr(slot_table), _ptr(ids), _ptr(w), _ptr(offsets), _ptr(pairs), _ptr(active),
                                   _ptr(n_active), _ptr(slots), _ptr(miss), _ptr(n_miss), _ptr(y), _ptr(ws),
                                   int(ws_bytes), _ptr(dev_err), _stream(stream)),
        "moe_route_expert_ffn")


def moe_slot_lookup(slot_table, active, n_active, pass_begin, pass_len, n_slots, slots, miss, n_miss, dev_err,
                    stream=None) -> None:
    _ck(lib().moe_slot_lookup(_ptr(slot_table), _ptr(active), _ptr(n_active), int(pass_begin), int(pass_len),
                              int(n_slots), _ptr(slots), _ptr(miss), _ptr(n_miss), _ptr(dev_err), _stream(stream)),
        "moe_slot_lookup")


def moe_install_slots(pool, slot_bytes, n_slots, host_rows, slots, side=None, done=None) -> None:
    """host_rows: sequence of pinned host addresses (ints); slots: host ints."""
    n = len(slots)
    rows = (C.c_void_p * max(n, 1))(*host_rows)
    sl = (C.c_int32 * max(n, 1))(*[int(s) for s in slots])
    ev = None if done is None else (done if isinstance(done, int) else done.cuda_event)
    _ck(lib().moe_install_slots(_ptr(pool), int(slot_bytes), int(n_slots), rows, sl, n, _stream(side), ev),
        "moe_install_slots")


def moe_expert_ffn(x, T, d, pool, n_slots, slot_table, ids, w, offsets, pairs, active, n_active, x_sorted,
                   pass_begin, pass_len, y_accum, ws, ws_bytes, dev_err, stream=None) -> None:
    _ck(lib().moe_expert_ffn(_ptr(x), int(T), C.byref(d), _ptr(pool), int(n_slots), _ptr(slot_table), _ptr(ids),
                             _ptr(w), _ptr(offsets), _ptr(pairs), _ptr(active), _ptr(n_active), _ptr(x_sorted),
                             int(pass_begin), int(pass_len), _ptr(y_accum), _ptr(ws), int(ws_bytes), _ptr(dev_err),
                             _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_noalloc(x, T, d, pool, n_slots, slot_table, ids, w, offsets, pairs, active, n_active,
                           pass_begin, pass_len, y_accum, dev_err, stream=None) -> None:
    """moe_expert_ffn with the library's own fixed scratch array (no workspace
    argument): for callers that cannot allocate device memory."""
    _ck(lib().moe_expert_ffn_noalloc(_ptr(x), int(T), C.byref(d), _ptr(pool), int(n_slots), _ptr(slot_table),
                                     _ptr(ids), _ptr(w), _ptr(offsets), _ptr(pairs), _ptr(active), _ptr(n_active),
                                     int(pass_begin), int(pass_len), _ptr(y_accum), _ptr(dev_err),
                                     _stream(stream)), "moe_expert_ffn_noalloc")


def moe_noalloc_scratch_bytes() -> int:
    return int(lib().moe_noalloc_scratch_bytes())


def moe_dequant_slot(pool, slot, d, out_fp32, out_bf16, stream=None) -> None:
    _ck(lib().moe_dequant_slot(_ptr(pool), int(slot), C.byref(d), _ptr(out_fp32), _ptr(out_bf16),
                               _stream(stream)), "moe_dequant_slot")


def moe_quantize_rows(w, rows, K, group, bits, proj, stream=None, gate_up_I=0) -> None:
    _ck(lib().moe_quantize_rows(_ptr(w), int(rows), int(K), int(group), int(bits), int(gate_up_I), _ptr(proj),
                                _stream(stream)), "moe_quantize_rows")


def moe_exp_portable(x, n, out, stream=None) -> None:
    _ck(lib().moe_exp_portable(_ptr(x), int(n), _ptr(out), _stream(stream)), "moe_exp_portable")


# ---------------------------------------------------------------------------
# host slot cache
# ---------------------------------------------------------------------------
class SlotCache:
    """moe_cache_*: one LRU per (size class, layer), host memory."""

    def __init__(self, E: int, n_layers: int, slots_per_layer: int, layer_class=None):
        self.E, self.n_layers, self.S = E, n_layers, slots_per_layer
        h = C.c_void_p()
        lc = None if layer_class is None else (C.c_int32 * n_layers)(*[int(c) for c in layer_class])
        _ck(lib().moe_cache_create(E, n_layers, lc, slots_per_layer, C.byref(h)), "moe_cache_create")
        self._h = h
        self._out_e = (C.c_int32 * E)()
        self._out_s = (C.c_int32 * E)()

    def close(self):
        if self._h:
            lib().moe_cache_destroy(self._h)
            self._h = None

    __del__ = close

    def table(self, layer: int):
        """Host expert -> slot table of the layer (a live ctypes view, length E)."""
        p = lib().moe_cache_table(self._h, layer)
        return (C.c_int32 * self.E).from_address(C.addressof(p.contents))

    def table_address(self, layer: int) -> int:
        return C.addressof(lib().moe_cache_table(self._h, layer).contents)

    def layer_base(self, layer: int) -> int:
        return int(lib().moe_cache_layer_base(self._h, layer))

    def class_slots(self, cls: int) -> int:
        return int(lib().moe_cache_class_slots(self._h, cls))

    def place(self, layer: int, experts, slots) -> None:
        n = len(experts)
        ea = (C.c_int32 * max(n, 1))(*[int(e) for e in experts])
        sa = (C.c_int32 * max(n, 1))(*[int(s) for s in slots])
        _ck(lib().moe_cache_place(self._h, layer, ea, sa, n), "moe_cache_place")

    def step(self, layer: int, pass_experts):
        """Returns (status, [(expert, slot), ...]) for the misses, ascending."""
        n = len(pass_experts)
        pa = (C.c_int32 * max(n, 1))(*[int(e) for e in pass_experts])
        nout = C.c_int32(0)
        st = lib().moe_cache_step(self._h, layer, pa, n, self._out_e, self._out_s, C.byref(nout))
        if st not in (MOE_OK, MOE_ERR_CAPACITY):
            _ck(st, "moe_cache_step")
        return st, [(self._out_e[i], self._out_s[i]) for i in range(nout.value)]

    def resident(self, layer: int) -> int:
        return int(lib().moe_cache_resident(self._h, layer))

    def reserve(self, layer: int, experts):
        """Returns [(expert, slot), ...] reserved for guessed copies."""
        n = len(experts)
        ea = (C.c_int32 * max(n, 1))(*[int(e) for e in experts])
        nout = C.c_int32(0)
        _ck(lib().moe_cache_reserve(self._h, layer, ea, n, self._out_e, self._out_s, C.byref(nout)),
            "moe_cache_reserve")
        return [(self._out_e[i], self._out_s[i]) for i in range(nout.value)]

    def commit(self, layer: int, slot: int) -> bool:
        """The guessed copy into `slot` landed; True if its expert entered the table."""
        ent = C.c_int32(0)
        _ck(lib().moe_cache_commit(self._h, layer, int(slot), C.byref(ent)), "moe_cache_commit")
        return bool(ent.value)

    def stats(self):
        h, m, e = C.c_int64(), C.c_int64(), C.c_int64()
        lib().moe_cache_stats(self._h, C.byref(h), C.byref(m), C.byref(e))
        return h.value, m.value, e.value


def moe_router_logits(x, T, W, bias, scale, E, H, logits, stream=None) -> None:
    _ck(lib().moe_router_logits(_ptr(x), int(T), _ptr(W), _ptr(bias), float(scale), int(E), int(H), _ptr(logits),
                                _stream(stream)), "moe_router_logits")


class Prefetch:
    """moe_prefetch_*: the guessed copies in flight, per layer."""

    def __init__(self, n_layers: int):
        h = C.c_void_p()
        _ck(lib().moe_prefetch_create(n_layers, C.byref(h)), "moe_prefetch_create")
        self._h = h

    def close(self):
        if self._h:
            lib().moe_prefetch_destroy(self._h)
            self._h = None

    __del__ = close

    def stats(self) -> dict:
        v = [C.c_int64() for _ in range(5)]
        lib().moe_prefetch_stats(self._h, *[C.byref(x) for x in v])
        return dict(zip(("guessed", "started", "entered", "wasted", "skipped_in_flight"), [x.value for x in v]))


def moe_decode_layer_ahead(cache: "SlotCache", pf: Prefetch, layer: int, ctx: LayerCtx, bufs: StepBuffers, x,
                           logits, T: int, L: float, y, stream, side, installed, guesses, gbufs: GuessBuffers,
                           ahead) -> int:
    """moe_decode_layer with guessed prefetch; guesses: [(layer, LayerCtx, logits tensor, top), ...] (0..2)."""
    n = C.c_int32(0)
    ev = installed if isinstance(installed, int) else installed.cuda_event
    ga = (Guess * max(len(guesses), 1))(*[Guess(int(gl), C.pointer(gc), _ptr(glog), int(top))
                                          for gl, gc, glog, top in guesses])
    _ck(lib().moe_decode_layer_ahead(cache._h, pf._h, int(layer), C.byref(ctx), C.byref(bufs), _ptr(x), _ptr(logits),
                                     int(T), float(L), _ptr(y), _stream(stream), _stream(side), ev, C.byref(n), ga,
                                     len(guesses), C.byref(gbufs), _stream(ahead)), "moe_decode_layer_ahead")
    return n.value


def moe_decode_layer(cache: "SlotCache", layer: int, ctx: LayerCtx, bufs: StepBuffers, x, logits, T: int, L: float,
                     y, stream, side, installed) -> int:
    """One decode layer through the native driver; returns experts installed."""
    n = C.c_int32(0)
    ev = installed if isinstance(installed, int) else installed.cuda_event
    _ck(lib().moe_decode_layer(cache._h, int(layer), C.byref(ctx), C.byref(bufs), _ptr(x), _ptr(logits), int(T),
                               float(L), _ptr(y), _stream(stream), _stream(side), ev, C.byref(n)),
        "moe_decode_layer")
    return n.value
