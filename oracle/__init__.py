"""CPU oracle for the streamed, quantized routed-expert FFN.

TEST INFRASTRUCTURE ONLY.  The test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or executes anything here, and nothing here imports the CUDA
library.  Arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation, fp32
where a float decides an integer); this module only marshals numpy arrays.

What each function follows on the pages is cited in ``oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, no CUDA)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))
    ):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        P = C.c_void_p
        i32, i64, u32, f32 = C.c_int32, C.c_int64, C.c_uint32, C.c_float
        sig = {
            "orc_exp_portable": (f32, [f32]),
            "orc_exp_portable_range": (None, [P, i64, P]),
            "orc_exp_portable_neg_bits": (None, [u32, i64, P]),
            "orc_route": (None, [P, i32, i32, i32, f32, P, P, P, P]),
            "orc_sort": (None, [P, i32, i32, i32, P, P, P, P]),
            "orc_slot_lookup": (None, [P, P, i32, i32, i32, i32, P, P, P, P]),
            "orc_bits_supported": (C.c_int, [i32]),
            "orc_row_bytes": (i64, [i32, i32]),
            "orc_row_groups": (i64, [i32, i32]),
            "orc_slot_layout": (None, [i32, i32, i32, i32, i32, P]),
            "orc_get_code": (i32, [P, i32, i32, i32, i32, i32]),
            "orc_set_code": (None, [P, i32, i32, i32, i32, i32, i32]),
            "orc_tile_bytes": (i64, [i32, i32, i32]),
            "orc_gate_up_row": (i32, [i32, i32]),
            "orc_quantize_rows": (None, [P, i32, i32, i32, i32, P]),
            "orc_dequant_rows": (None, [P, i32, i32, i32, i32, P]),
            "orc_dequant_slot": (None, [P, i32, i32, i32, i32, i32, P, P]),
            "orc_expert_ffn": (None, [P, i32, i32, i32, i32, i32, i32, P, P, P, P, i32, P]),
            "orc_lru_step": (i32, [i32, i32, i32, P, P, P, P, P, i32, P, P]),
            "orc_bf16_to_f32": (f32, [C.c_uint16]),
            "orc_f32_to_bf16": (C.c_uint16, [f32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


# --------------------------------------------------------------------------
# exp used by routing
# --------------------------------------------------------------------------
def exp_portable(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    flat = np.ascontiguousarray(x.reshape(-1))
    out = np.empty_like(flat)
    lib().orc_exp_portable_range(_p(flat), flat.size, _p(out))
    return out.reshape(x.shape)


def exp_portable_neg_bits(start: int, n: int) -> np.ndarray:
    """exp of the floats with bit patterns 0x80000000 | (start + i), i < n."""
    out = np.empty(n, dtype=np.float32)
    lib().orc_exp_portable_neg_bits(start, n, _p(out))
    return out


# --------------------------------------------------------------------------
# stages 1-3
# --------------------------------------------------------------------------
def route(logits: np.ndarray, k: int, L: float = 0.0, slot_table: np.ndarray | None = None):
    """Returns (ids int32 [T,k], w float64 [T,k], u float32 [T,E])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    u = np.empty((T, E), np.float32)
    st = None
    if slot_table is not None:
        st = np.ascontiguousarray(slot_table, dtype=np.int32)
        assert st.shape == (E,)
    lib().orc_route(_p(logits), T, E, k, float(L), _p(st) if st is not None else None, _p(ids), _p(w), _p(u))
    return ids, w, u


def router_logits(x_bf16: np.ndarray, W_bf16: np.ndarray, bias, scale: float) -> np.ndarray:
    """logits[t][e] = scale * sum_h x[t][h] W[e][h] + bias[e], in double from
    the bf16 inputs: a layer's router evaluated on a hidden state (RFC "How
    the prototype works", item "Reads": the next layers' routers run on the
    current hidden states to guess their experts)."""
    x = (np.ascontiguousarray(x_bf16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    W = (np.ascontiguousarray(W_bf16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    out = float(scale) * (x @ W.T)
    if bias is not None:
        out += np.asarray(bias, np.float32).astype(np.float64)[None, :]
    return out


def route_shared(logits: np.ndarray, k: int, n_shared: int, shared_w=None, L: float = 0.0,
                 slot_table: np.ndarray | None = None):
    """route(), then every token's always-on shared experts (BigMoeOnEdge
    docs/limitations.md, "Limitations", "Shared experts stay resident": the
    shared expert runs for every token).  Shared expert s of a layer with E
    routed experts has id E + s and weight shared_w[t] (1 when None) for
    every token; the top-k weights stay normalised over the top-k alone.
    Returns (ids int32 [T, k + n_shared], w float64 [T, k + n_shared], u)."""
    ids, w, u = route(logits, k, L, slot_table)
    T, E = np.asarray(logits).shape
    sid = np.broadcast_to(np.arange(E, E + n_shared, dtype=np.int32), (T, n_shared))
    if shared_w is None:
        sw = np.ones((T, n_shared), np.float64)
    else:
        sw = np.repeat(np.asarray(shared_w, np.float32).astype(np.float64)[:, None], n_shared, axis=1)
    return (np.ascontiguousarray(np.concatenate([ids, sid], axis=1), dtype=np.int32),
            np.ascontiguousarray(np.concatenate([w, sw], axis=1)), u)


def sort(ids: np.ndarray, E: int):
    """Returns (offsets [E+1], pairs [T*k], active [n_active])."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, np.int32)
    pairs = np.empty(T * k, np.int32)
    active = np.empty(E, np.int32)
    na = np.zeros(1, np.int32)
    lib().orc_sort(_p(ids), T, k, E, _p(offsets), _p(pairs), _p(active), _p(na))
    return offsets, pairs, active[: int(na[0])].copy()


def slot_lookup(table: np.ndarray, active: np.ndarray, pass_begin: int, pass_len: int, n_slots: int):
    """Returns (slots, miss, bad)."""
    table = np.ascontiguousarray(table, dtype=np.int32)
    active = np.ascontiguousarray(active, dtype=np.int32)
    n = max(0, min(pass_begin + pass_len, active.size) - pass_begin)
    slots = np.empty(max(n, 1), np.int32)
    miss = np.empty(max(n, 1), np.int32)
    nm = np.zeros(1, np.int32)
    bad = np.zeros(1, np.int32)
    lib().orc_slot_lookup(_p(table), _p(active), active.size, pass_begin, pass_len, n_slots, _p(slots),
                          _p(miss), _p(nm), _p(bad))
    return slots[:n].copy(), miss[: int(nm[0])].copy(), int(bad[0])


# --------------------------------------------------------------------------
# format, quantization, dequantization
# --------------------------------------------------------------------------
def row_bytes(K: int, b: int) -> int:
    return int(lib().orc_row_bytes(K, b))


def row_groups(K: int, g: int) -> int:
    return int(lib().orc_row_groups(K, g))


def slot_layout(H: int, I: int, g: int, b_gu: int, b_d: int):
    """([gate_up offset, down offset, gate_up tile bytes, down tile bytes], slot bytes)."""
    off = np.zeros(5, np.int64)
    lib().orc_slot_layout(H, I, g, b_gu, b_d, _p(off))
    return [int(v) for v in off[:4]], int(off[4])


def tile_bytes(K: int, g: int, b: int) -> int:
    return int(lib().orc_tile_bytes(K, g, b))


def slot_bytes(H: int, I: int, g: int, b_gu: int, b_d: int) -> int:
    return slot_layout(H, I, g, b_gu, b_d)[1]


def get_code(proj: np.ndarray, K: int, g: int, row: int, k: int, b: int) -> int:
    """Code of input k of row `row` of a projection (bytes of all its tiles)."""
    proj = np.ascontiguousarray(proj, dtype=np.uint8)
    return int(lib().orc_get_code(_p(proj), K, g, row, k, b))


def set_code(proj: np.ndarray, K: int, g: int, row: int, k: int, b: int, q: int) -> None:
    assert proj.dtype == np.uint8 and proj.flags["C_CONTIGUOUS"]
    lib().orc_set_code(_p(proj), K, g, row, k, b, q)


def gate_up_row(R: int, I: int) -> int:
    """Storage row of logical gate/up row R."""
    return int(lib().orc_gate_up_row(R, I))


def gate_up_order(I: int) -> np.ndarray:
    """order[p] = logical gate/up row stored at storage row p."""
    order = np.empty(2 * I, np.int64)
    for R in range(2 * I):
        order[gate_up_row(R, I)] = R
    return order


def quantize_rows(w: np.ndarray, g: int, b: int) -> np.ndarray:
    """w fp32 [rows, K] (storage order, rows a multiple of 16) -> the
    projection's bytes, uint8 [rows/16, tile_bytes] (see oracle.c)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, K = w.shape
    assert rows % 16 == 0, "rows come in tiles of 16"
    proj = np.zeros((rows // 16, tile_bytes(K, g, b)), np.uint8)
    lib().orc_quantize_rows(_p(w), rows, K, g, b, _p(proj))
    return proj


def dequant_rows(proj: np.ndarray, rows: int, K: int, g: int, b: int) -> np.ndarray:
    proj = np.ascontiguousarray(proj, dtype=np.uint8)
    out = np.empty((rows, K), np.float32)
    lib().orc_dequant_rows(_p(proj), rows, K, g, b, _p(out))
    return out


def build_slot(w_gu: np.ndarray, w_d: np.ndarray, g: int, b_gu: int, b_d: int) -> np.ndarray:
    """Quantize one expert (w_gu [2I,H], w_d [H,I], fp32) into its slot bytes."""
    I2, H = w_gu.shape
    I = I2 // 2
    assert w_d.shape == (H, I)
    off, nbytes = slot_layout(H, I, g, b_gu, b_d)
    slot = np.zeros(nbytes, np.uint8)
    pg = quantize_rows(np.ascontiguousarray(w_gu[gate_up_order(I)]), g, b_gu)
    pd = quantize_rows(w_d, g, b_d)
    slot[off[0]: off[0] + pg.size] = pg.reshape(-1)
    slot[off[1]: off[1] + pd.size] = pd.reshape(-1)
    return slot


def dequant_slot(slot: np.ndarray, H: int, I: int, g: int, b_gu: int, b_d: int):
    """Slot bytes -> (gate_up fp32 [2I,H], down fp32 [H,I]); deq = fma(s, q, b)."""
    slot = np.ascontiguousarray(slot, dtype=np.uint8)
    gu = np.empty((2 * I, H), np.float32)
    dn = np.empty((H, I), np.float32)
    lib().orc_dequant_slot(_p(slot), H, I, g, b_gu, b_d, _p(gu), _p(dn))
    return gu, dn


# --------------------------------------------------------------------------
# stages 4-5
# --------------------------------------------------------------------------
def expert_ffn(x_bf16: np.ndarray, H: int, I: int, g: int, b_gu: int, b_d: int, ids: np.ndarray, w: np.ndarray,
               expert_slots, tokens=None) -> np.ndarray:
    """y[t] = sum_j w[t,j] * W_d silu(W_g x_t) * (W_u x_t), in double.

    x_bf16: uint16 bf16 bit patterns [T, H].  expert_slots: sequence, entry e
    = slot bytes (uint8) of expert e (None for experts never routed).
    tokens: subset of token indices (default all).  Returns [n_tok, H] float64.
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    T = x.shape[0]
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    k = ids.shape[1]
    w = np.ascontiguousarray(w, dtype=np.float64)
    tok = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    keep = []
    ptrs = (C.c_void_p * len(expert_slots))()
    for e, s in enumerate(expert_slots):
        if s is None:
            ptrs[e] = None
        else:
            s = np.ascontiguousarray(s, dtype=np.uint8)
            keep.append(s)
            ptrs[e] = s.ctypes.data
    for t in tok:
        for e in ids[t]:
            assert expert_slots[int(e)] is not None, f"expert {int(e)} has no slot bytes"
    y = np.empty((tok.size, H), np.float64)
    lib().orc_expert_ffn(_p(x), H, I, g, b_gu, b_d, k, C.cast(ptrs, C.c_void_p), _p(ids), _p(w), _p(tok),
                         tok.size, _p(y))
    return y


# --------------------------------------------------------------------------
# host slot cache model
# --------------------------------------------------------------------------
class LruModel:
    """One LRU per (size class, layer) over that layer's own slot range."""

    def __init__(self, E: int, n_slots: int, slot_base: int = 0):
        self.E, self.n_slots, self.base = E, n_slots, slot_base
        self.table = np.full(E, -1, np.int32)
        self.owner = np.full(n_slots, -1, np.int32)
        self.stamp = np.zeros(n_slots, np.int64)
        self.clock = np.zeros(1, np.int64)

    def place(self, experts, slots) -> None:
        """Initial residency: expert experts[i] in slot slots[i] (absolute id)."""
        for e, s in zip(experts, slots):
            self.table[e] = s
            self.owner[s - self.base] = e
            self.clock[0] += 1
            self.stamp[s - self.base] = self.clock[0]  # more recent than any empty slot

    def step(self, pass_experts):
        """Touch hits, assign misses; returns the slot given to each miss, in order."""
        pe = np.ascontiguousarray(pass_experts, dtype=np.int32)
        assigned = np.empty(max(pe.size, 1), np.int32)
        na = np.zeros(1, np.int32)
        fail = lib().orc_lru_step(self.E, self.n_slots, self.base, _p(self.table), _p(self.owner),
                                  _p(self.stamp), _p(self.clock), _p(pe), pe.size, _p(assigned), _p(na))
        return assigned[: int(na[0])].copy(), int(fail)
