"""Per-layer driver of the streamed expert FFN over the C ABI.

Sequencing only: every step below is one libmoe call (or a plain copy).
  decode layer:  route -> sort -> slot lookup -> (misses to host, LRU step,
                 pinned installs on a side stream, table upload) -> FFN
  prefill layer: route (L = 0) -> sort -> for each pass of <= 64 active
                 experts: lookup -> installs -> FFN   (RFC "How the prototype
                 works", items "Reads" and "Prefill")
When every expert of a layer is resident the layer never synchronises with
the host (RFC: "When every expert is resident, layers never synchronize with
the host").  Layers are grouped into size classes by slot byte size, one
device pool and one LRU range per (class, layer) (1bit-MONSTER PR #137).
Always-on shared experts (BigMoeOnEdge docs/limitations.md, "Shared experts
stay resident") get pinned slots after the class's LRU ranges and run in the
same FFN launch as the routed experts (moe_route_shared widens the layer).
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import ops

PASS_EXPERTS = 64  # RFC / PR #50717: sorted prefill runs 64 experts at a time


@dataclass
class LayerSpec:
    desc: ops.LayerDesc
    bank: torch.Tensor            # pinned uint8 [rows, slot_bytes] of this layer's class
    bank_row: list                # expert e -> row of `bank`
    shared: torch.Tensor | None = None  # uint8 [n_shared, slot_bytes]: the layer's shared experts


def quantize_bank_gpu(E: int, desc: ops.LayerDesc, seed: int, device="cuda", std: float = 0.02) -> torch.Tensor:
    """Pinned uint8 [E, slot_bytes]: expert e = N(0, std) weights (seeded torch
    generator) quantised on the GPU by moe_quantize_rows into the slot format."""
    from . import synth

    lay = ops.moe_slot_layout(desc)
    sb = int(lay.slot_bytes)
    H, I, g = desc.H, desc.I, desc.group
    bank = torch.empty((E, sb), dtype=torch.uint8).pin_memory()
    slot = torch.zeros(sb, dtype=torch.uint8, device=device)
    for e in range(E):
        w_gu, w_d = synth.expert_weights_torch(seed, e, H, I, device, std)
        base = slot.data_ptr()
        ops.moe_quantize_rows(w_gu, 2 * I, H, g, desc.bits_gu, base + lay.gate_up, gate_up_I=I)
        ops.moe_quantize_rows(w_d, H, I, g, desc.bits_down, base + lay.down)
        bank[e].copy_(slot, non_blocking=False)
    return bank


class Streamer:
    def __init__(self, layers: list[LayerSpec], slots_per_layer: int, max_tokens: int, device="cuda",
                 stream: torch.cuda.Stream | None = None, n_shared: int = 0):
        self.layers = layers
        self.n_layers = len(layers)
        self.device = torch.device(device)
        self.E = layers[0].desc.E
        self.k = layers[0].desc.k
        self.H = layers[0].desc.H
        assert all(l.desc.E == self.E and l.desc.H == self.H for l in layers)
        self.ns = n_shared
        assert n_shared == 0 or all(l.shared is not None and l.shared.shape[0] == n_shared for l in layers)
        self.Ew, self.kw = self.E + n_shared, self.k + n_shared  # the widened layer
        self.wdesc = [ops.widened(l.desc, n_shared) for l in layers]
        self.S = slots_per_layer
        self.max_tokens = max_tokens
        self.stream = stream or torch.cuda.current_stream(self.device)
        self.side = torch.cuda.Stream(self.device)
        self.installed = torch.cuda.Event()
        # size classes
        sizes = []
        self.layer_class = []
        for l in layers:
            sb = ops.moe_slot_bytes(l.desc)
            if sb not in sizes:
                sizes.append(sb)
            self.layer_class.append(sizes.index(sb))
        self.class_bytes = sizes
        self.cache = ops.SlotCache(self.E, self.n_layers, self.S, self.layer_class)
        # per class: the LRU's slots, then n_shared pinned slots per layer of the class
        self.pools = []
        self.class_n_slots = []
        for c, sb in enumerate(sizes):
            n = self.cache.class_slots(c) + n_shared * self.layer_class.count(c)
            self.pools.append(torch.empty(n * sb, dtype=torch.uint8, device=self.device))
            self.class_n_slots.append(n)
        # device tables + pinned mirrors (routed experts, then the shared ones)
        self.table_dev = torch.full((self.n_layers, self.Ew), -1, dtype=torch.int32, device=self.device)
        self.table_pin = torch.full((self.n_layers, self.Ew), -1, dtype=torch.int32).pin_memory()
        for l in range(self.n_layers) if n_shared else ():
            c = self.layer_class[l]
            first = self.cache.class_slots(c) + n_shared * self.layer_class[:l].count(c)
            sb = self.class_bytes[c]
            for s_ in range(n_shared):
                self.pools[c][(first + s_) * sb: (first + s_ + 1) * sb].copy_(layers[l].shared[s_])
                self.table_pin[l, self.E + s_] = first + s_
        self.table_dev.copy_(self.table_pin)
        # per-call buffers (widened layer)
        T, E, k = max_tokens, self.Ew, self.kw
        self.ids = torch.empty((T, k), dtype=torch.int32, device=self.device)
        self.w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=self.device)
        self.pairs = torch.empty(max(T * k, 1), dtype=torch.int32, device=self.device)
        # meta: [n_active, n_miss, active[E], miss[E]] -> one small D2H per layer
        self.meta = torch.zeros(2 + 2 * E, dtype=torch.int32, device=self.device)
        self.meta_pin = torch.zeros(2 + 2 * E, dtype=torch.int32).pin_memory()
        self.slots = torch.empty(E, dtype=torch.int32, device=self.device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=self.device)
        ws = max(ops.moe_workspace_bytes(d, T) for d in self.wdesc)
        self.ws_bytes = ws
        self.ws = torch.zeros(ws, dtype=torch.uint8, device=self.device)
        self.x_sorted = None
        self.y = torch.zeros((T, self.H), dtype=torch.float32, device=self.device)
        self.installed_bytes = 0
        self.installs = 0
        self.launches = 0          # libmoe kernel launches issued (for reporting)
        self._paths = {}           # (layer, T, sorted x) -> moe_ffn_kernel_path
        # native per-layer driver state
        self.installed.record(self.side)  # materialise the event
        bf16 = any(l.desc.bits_gu == 16 or l.desc.bits_down == 16 for l in layers)
        if max_tokens >= 32 or bf16:  # the tensor-core grouped GEMM (batched decode, BF16 experts) reads sorted x
            self.x_sorted = torch.empty((max_tokens * self.kw, self.H), dtype=torch.uint16, device=self.device)
        self._bufs = ops.StepBuffers(self.ids.data_ptr(), self.w.data_ptr(), self.offsets.data_ptr(),
                                     self.pairs.data_ptr(), self.meta.data_ptr(), self.meta_pin.data_ptr(),
                                     self.slots.data_ptr(), self.dev_err.data_ptr(), self.ws.data_ptr(),
                                     self.ws_bytes, max_tokens,
                                     self.x_sorted.data_ptr() if self.x_sorted is not None else None)
        self._ctx = []
        self._rows = []
        for l, spec in enumerate(layers):
            rows = (C.c_void_p * self.E)(*[self._row_addr(l, e) for e in range(self.E)])
            self._rows.append(rows)
            self._ctx.append(ops.LayerCtx(C.pointer(spec.desc), self.pools[self.layer_class[l]].data_ptr(),
                                          self.class_n_slots[self.layer_class[l]],
                                          self.class_bytes[self.layer_class[l]], self.table_dev[l].data_ptr(),
                                          self.table_pin[l].data_ptr(), rows, n_shared, None))
        self.ffn_events = None     # list to collect (start, end) CUDA events around FFN calls
        # guessed prefetch (moe_decode_layer_ahead): its own copy stream, state and buffers
        self.prefetch = ops.Prefetch(self.n_layers)
        self.ahead = torch.cuda.Stream(self.device)
        stride = max(max_tokens * self.k, 1)
        self.g_ids = torch.empty(2 * stride, dtype=torch.int32, device=self.device)
        self.g_w = torch.empty(2 * stride, dtype=torch.float32, device=self.device)
        self.g_ids_pin = torch.empty(2 * stride, dtype=torch.int32).pin_memory()
        self._gbufs = ops.GuessBuffers(self.g_ids.data_ptr(), self.g_w.data_ptr(), self.g_ids_pin.data_ptr(), stride)

    # -- views into meta --------------------------------------------------
    def _n_active(self):
        return self.meta[0:1]

    def _n_miss(self):
        return self.meta[1:2]

    def _active(self):
        return self.meta[2: 2 + self.Ew]

    def _miss(self):
        return self.meta[2 + self.Ew: 2 + 2 * self.Ew]

    # -- residency ----------------------------------------------------------
    def pool_of(self, layer: int) -> torch.Tensor:
        return self.pools[self.layer_class[layer]]

    def n_slots_of(self, layer: int) -> int:
        return self.class_n_slots[self.layer_class[layer]]

    def _row_addr(self, layer: int, e: int) -> int:
        spec = self.layers[layer]
        row = spec.bank_row[e]
        return spec.bank.data_ptr() + row * spec.bank.shape[1]

    def _upload_table(self, layer: int, stream) -> None:
        tab = self.cache.table(layer)
        C.memmove(self.table_pin[layer].data_ptr(), C.addressof(tab), 4 * self.E)
        with torch.cuda.stream(stream):
            self.table_dev[layer].copy_(self.table_pin[layer], non_blocking=True)

    def place(self, layer: int, experts, slots_rel=None) -> None:
        """Make `experts` resident in layer `layer` (slots relative to the
        layer's range; default 0, 1, ...), copying their rows synchronously."""
        base = self.cache.layer_base(layer)
        rel = list(range(len(experts))) if slots_rel is None else list(slots_rel)
        self.cache.place(layer, experts, [base + s for s in rel])
        sb = self.class_bytes[self.layer_class[layer]]
        ops.moe_install_slots(self.pool_of(layer), sb, self.n_slots_of(layer),
                              [self._row_addr(layer, e) for e in experts], [base + s for s in rel],
                              self.side, None)
        self._upload_table(layer, self.side)
        self.side.synchronize()

    def fully_resident(self, layer: int) -> bool:
        return self.cache.resident(layer) >= self.E

    def _install_pass(self, layer: int, pass_experts) -> int:
        pass_experts = [e for e in pass_experts if e < self.E]  # shared experts stay where they are
        st, inst = self.cache.step(layer, pass_experts)
        if st != ops.MOE_OK:
            raise ops.MoeError(st, f"slot cache step (layer {layer})")
        if inst:
            sb = self.class_bytes[self.layer_class[layer]]
            ops.moe_install_slots(self.pool_of(layer), sb, self.n_slots_of(layer),
                                  [self._row_addr(layer, e) for e, _ in inst], [s for _, s in inst], self.side, None)
            self._upload_table(layer, self.side)
            self.installed.record(self.side)
            self.stream.wait_event(self.installed)
            self.installed_bytes += sb * len(inst)
            self.installs += len(inst)
        return len(inst)

    # -- stages -------------------------------------------------------------
    def route_sort(self, layer: int, x, logits, T: int, L: float = 0.0, want_sorted_x: bool = False):
        d, dw = self.layers[layer].desc, self.wdesc[layer]
        s = self.stream
        if self.ns:
            ops.moe_route_shared(logits, T, d, L, self.table_dev[layer], self.ns, None, self.ids, self.w, s)
        else:
            ops.moe_route(logits, T, d, L, self.table_dev[layer], self.ids, self.w, s)
        self.launches += 1
        xs = None
        if want_sorted_x:
            if self.x_sorted is None or self.x_sorted.numel() < T * self.kw * self.H:
                self.x_sorted = torch.empty((self.max_tokens * self.kw, self.H), dtype=torch.uint16,
                                            device=self.device)
            xs = self.x_sorted
        ops.moe_sort(self.ids, x if want_sorted_x else None, T, dw, self.offsets, self.pairs, self._active(),
                     self._n_active(), xs, self.ws, self.ws_bytes, s)
        self.launches += (1 if T * self.kw <= 1024 else 3) + (1 if want_sorted_x else 0)

    def ffn(self, layer: int, x, T: int, pass_begin: int, pass_len: int, y) -> None:
        d = self.wdesc[layer]
        ev = None
        if self.ffn_events is not None:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(self.stream)
        self.launches += 2 if T <= 64 else 3
        tc = self.uses_tc(layer, T)
        ops.moe_expert_ffn(x, T, d, self.pool_of(layer), self.n_slots_of(layer), self.table_dev[layer], self.ids,
                           self.w, self.offsets, self.pairs, self._active(), self._n_active(),
                           self.x_sorted if tc else None, pass_begin, pass_len, y, self.ws, self.ws_bytes,
                           self.dev_err, self.stream)
        if ev is not None:
            ev[1].record(self.stream)
            self.ffn_events.append(ev)

    def uses_tc(self, layer: int, T: int) -> bool:
        """Whether the layer's FFN over T tokens runs on the tensor-core grouped
        GEMM (which reads x sorted by expert) when given sorted x."""
        key = (layer, T, "tc")
        v = self._paths.get(key)
        if v is None:
            v = self._paths[key] = ops.moe_ffn_kernel_path(self.wdesc[layer], T, True) == ops.MOE_PATH_TC_PREFILL
        return v

    def _ffn_launches(self, layer: int, T: int, pass_len: int) -> int:
        """Kernels one moe_expert_ffn call over pass_len experts launches."""
        d = self.wdesc[layer]
        tc = self.uses_tc(layer, T)
        key = (layer, T, tc)
        path = self._paths.get(key)
        if path is None:
            path = self._paths[key] = ops.moe_ffn_kernel_path(d, T, tc)
        if path == 0:
            return 1  # the fused decode kernel
        if path == 2:  # gate/up + down per sub-range of 64 experts, then the combine
            return 2 * -(-min(pass_len, self.Ew) // 64) + 1
        return 3

    def _decode_launches(self, layer: int, T: int, full: bool, n_installed: int, guessing: bool = False) -> int:
        d = self.layers[layer].desc
        tc = self.uses_tc(layer, T)
        if T == 1 and not tc:
            if not self.ns and full and not guessing and d.E <= 1024 and self._ffn_launches(layer, T, self.Ew) == 1:
                return 1  # moe_route_expert_ffn: every stage in the FFN launch
            n = 1  # moe_route_sort_lookup
        else:
            n = 1 + (1 if T * self.kw <= 1024 else 3) + (1 if tc else 0) + (0 if full else 1)  # route, sort, lookup
        if n_installed:  # resident experts, then the installed ones
            return n + self._ffn_launches(layer, T, self.kw * T) + self._ffn_launches(layer, T, n_installed)
        return n + self._ffn_launches(layer, T, self.Ew)

    def decode_layer(self, layer: int, x, logits, T: int, L: float = 0.0, y=None):
        """One decode layer (T <= 64 tokens) through the native driver
        (moe_decode_layer); returns y fp32 [T, H] (device)."""
        y = self.y[:T] if y is None else y
        full = self.cache.resident(layer) >= self.E
        n = ops.moe_decode_layer(self.cache, layer, self._ctx[layer], self._bufs, x, logits, T, L, y, self.stream,
                                 self.side, self.installed)
        if n:
            self.installs += n
            self.installed_bytes += n * self.class_bytes[self.layer_class[layer]]
        self.launches += self._decode_launches(layer, T, full, n)
        return y

    def decode_layer_ahead(self, layer: int, x, logits, T: int, L: float = 0.0, guesses=(), y=None):
        """decode_layer with guessed prefetch (moe_decode_layer_ahead).
        guesses: up to two (later layer, logits [T, E] device[, top]) tuples,
        each that layer's router evaluated on this layer's hidden state; top =
        how many of each token's best guesses to read ahead (default all k)."""
        y = self.y[:T] if y is None else y
        full = self.cache.resident(layer) >= self.E
        g = [(gu[0], self._ctx[gu[0]], gu[1], gu[2] if len(gu) > 2 else 0) for gu in guesses]
        n = ops.moe_decode_layer_ahead(self.cache, self.prefetch, layer, self._ctx[layer], self._bufs, x, logits, T,
                                       L, y, self.stream, self.side, self.installed, g, self._gbufs, self.ahead)
        if n:
            self.installs += n
            self.installed_bytes += n * self.class_bytes[self.layer_class[layer]]
        self.launches += self._decode_launches(layer, T, full, n, guessing=bool(g)) + len(g)
        return y

    def decode_layer_steps(self, layer: int, x, logits, T: int, L: float = 0.0, y=None):
        """Same as decode_layer, one ABI call at a time from Python."""
        y = self.y[:T] if y is None else y
        s = self.stream
        d0 = self.layers[layer].desc
        self.route_sort(layer, x, logits, T, L, want_sorted_x=self.uses_tc(layer, T))
        if not self.fully_resident(layer):
            d = self.layers[layer].desc
            ops.moe_slot_lookup(self.table_dev[layer], self._active(), self._n_active(), 0, self.Ew,
                                self.n_slots_of(layer), self.slots, self._miss(), self._n_miss(), self.dev_err, s)
            self.launches += 1
            with torch.cuda.stream(s):
                self.meta_pin.copy_(self.meta, non_blocking=True)
            s.synchronize()
            na = int(self.meta_pin[0])
            act = self.meta_pin[2: 2 + na].tolist()
            self._install_pass(layer, act)
            del d
        with torch.cuda.stream(s):
            y.zero_()
        self.ffn(layer, x, T, 0, self.Ew, y)
        return y

    def prefill_layer(self, layer: int, x, logits, T: int, y=None):
        """One prefill chunk: passes of <= 64 active experts; returns y."""
        y = self.y[:T] if y is None else y
        s = self.stream
        d0 = self.layers[layer].desc
        self.route_sort(layer, x, logits, T, 0.0, want_sorted_x=self.uses_tc(layer, T))
        with torch.cuda.stream(s):
            y.zero_()
            self.meta_pin.copy_(self.meta, non_blocking=True)
        s.synchronize()
        na = int(self.meta_pin[0])
        active = self.meta_pin[2: 2 + na].tolist()
        resident = self.fully_resident(layer)
        for p in range(0, na, PASS_EXPERTS):
            pe = active[p: p + PASS_EXPERTS]
            if not resident:
                # every pass synchronises: its slots come from the host LRU
                ops.moe_slot_lookup(self.table_dev[layer], self._active(), self._n_active(), p, PASS_EXPERTS,
                                    self.n_slots_of(layer), self.slots, self._miss(), self._n_miss(), self.dev_err,
                                    s)
                self.launches += 1
                s.synchronize()  # previous pass's FFN done before its slots can be reused
                self._install_pass(layer, pe)
            self.ffn(layer, x, T, p, PASS_EXPERTS, y)
        return y

    def check_dev_err(self) -> int:
        """The device error word (MOE_DEV_ERR_* bits).  After a wait that ran
        out, the whole workspace (its control block and the tagged h words
        that carry over between calls) is zeroed before any later call."""
        v = int(self.dev_err.item())
        if v & ops.DEV_ERR_TIMEOUT:
            self.ws.zero_()
        return v
