"""Benchmark of the streamed, quantized routed-expert FFN on B200.

Default workload (N=1): Flash-Next-like decode, 48 layers x 512 experts,
top-10, hidden 2048, expert intermediate 512, SwiGLU, 3-bit affine g64 with
bf16 scale/bias, 1 token per step, 192 slots per layer; misses installed from
pinned host memory before compute.  A step = one token through all 48 layers
of the whole path (route, sort, slot lookup, installs, dequant+SwiGLU FFN,
combine).  Inputs are synthetic (seeded); the expert bank is drawn on the GPU
and quantised by the library.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--config decode|coder|prefill|tiny]
Under torchrun each rank runs an independent replica (its own token stream):
weak scaling, no collective on the data path.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "expert-FFN HBM GB/s & decode tok/s-equiv; prefill TFLOP/s; % of B200 roofline"


def max_over_ranks(values, device=None):
    """Element-wise max of `values` over the default process group (the
    values themselves without one): every rank gets the slowest rank's times."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the ncu capture recorded in
    profiles/traffic.txt, or None when the kernel's sources changed since."""
    import hashlib

    try:
        for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
            if line.startswith("#") or not line.strip():
                continue
            f = dict(kv.split("=", 1) for kv in line.split())
            if f.get("kernel") != kernel:
                continue
            m = hashlib.sha256()
            for src in f["sources"].split(","):
                with open(os.path.join(ROOT, "streamed_quantized_expert_b200", "csrc", src), "rb") as fh:
                    m.update(fh.read())
            return int(f["bytes"]) if m.hexdigest()[:16] == f["source_sha256"] else None
    except Exception:
        return None
    return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


CONFIGS = {
    # name: (layers, E, k, H, I, g, bits_gu, bits_down, T, slots_per_layer, description)
    "decode": (48, 512, 10, 2048, 512, 64, 3, 3, 1, 192,
               "Flash-Next-like decode: 48 layers x 512 experts, top-10, H 2048, I 512, SwiGLU, 3-bit g64, "
               "1 token/step, 192 slots/layer, misses installed from pinned host"),
    "coder": (48, 128, 8, 2048, 768, 64, 4, 4, 64, 128,
              "Coder-30B-like batched decode: 48 layers x 128 experts, top-8, H 2048, I 768, 4-bit g64, "
              "64 tokens/step, all 128 experts resident"),
    "tiny": (1, 8, 2, 64, 32, 32, 4, 4, 4, 8, "tiny MoE layer: 8 experts, top-2, H 64, I 32, 4-bit g32, 4 tokens"),
    "decode_shared": (48, 512, 10, 2048, 512, 64, 3, 3, 1, 192,
                      "Flash-Next-like decode with one always-on shared expert per layer (same shape, pinned slot, "
                      "run in the routed experts' FFN launch): 48 layers x 512 routed experts, top-10, H 2048, I 512, "
                      "3-bit g64, 1 token/step, 192 slots/layer, misses installed from pinned host"),
    "decode_resident": (48, 512, 10, 2048, 512, 64, 3, 3, 1, 512,
                        "Flash-Next-like decode with every expert resident: 48 layers x 512 experts, top-10, H 2048, "
                        "I 512, 3-bit g64, 1 token/step, 512 slots/layer (34 GB of slots); no layer synchronises "
                        "with the host, so each step is one CUDA graph of the 48 layers' moe_decode_layer calls"),
    "decode_mixed": (48, 512, 10, 2048, 512, 64, 4, 4, 1, 128,
                     "mixed size classes decode with cache-aware substitution: Flash-Next-like shapes, 4-bit "
                     "gate/up, 6-bit down on layers l % 4 == 0 (2 slot size classes), 1 token/step, 128 slots/layer "
                     "(25% resident), L = 0.15, misses installed from pinned host"),
}
# token counts of a configuration's batch sweep (besides its own T), FFN-only
SWEEP = {"coder": (1, 8, 16, 32)}
# per-layer widths and the substitution strength of the decode configurations (default: uniform, L = 0)
DECODE_EXTRA = {"decode_mixed": {"bits": lambda l: (4, 6) if l % 4 == 0 else (4, 4), "L": 0.15},
                "decode_shared": {"n_shared": 1},
                "decode_resident": {"graph_step": True}}

# Prefill chunks: every expert of every layer resident (the metric is the expert
# FFN's tensor-core rate; installs are PCIe-bound and reported by decode).
# name: (layers, E, k, H, I, g, bits(layer) -> (gate/up, down), T, description)
PREFILL = {
    "prefill": (48, 512, 10, 2048, 512, 64, lambda l: (3, 3), 1024,
                "Flash-Next-like prefill: 48 layers x 512 experts, top-10, H 2048, I 512, SwiGLU, 3-bit g64, "
                "1024-token chunk, passes of 64 active experts, tcgen05 grouped GEMM"),
    "prefill_bf16": (48, 128, 8, 2048, 768, 64, lambda l: (16, 16), 1024,
                     "Coder-30B-like prefill with unquantized BF16 experts: 48 layers x 128 experts, top-8, H 2048, "
                     "I 768, SwiGLU, bf16 weights (16-bit slots), 1024-token chunk, tcgen05 grouped GEMM"),
    "prefill_mixed": (48, 512, 10, 2048, 512, 64, lambda l: (4, 6) if l % 4 == 0 else (4, 4), 4096,
                      "mixed size classes prefill: Flash-Next-like shapes, 4-bit gate/up, 6-bit down on layers "
                      "l % 4 == 0 (2 slot size classes), 4096-token chunk, passes of 64 active experts"),
}


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx = float(f[2])
                except ValueError:
                    continue
                for n, v in zip(names, f[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
# The mixed-class configuration as one sequence: a prefill chunk through the
# 25%-resident two-class cache (passes of 64 active experts, installs between
# passes), then decode steps with cache-aware substitution from the cache the
# prefill left.
# name: (layers, E, k, H, I, g, bits(layer), prefill T, decode steps, slots per layer, L, description)
SEQUENCE = {
    "mixed_sequence": (48, 512, 10, 2048, 512, 64, lambda l: (4, 6) if l % 4 == 0 else (4, 4), 4096, 256, 128, 0.15,
                       "mixed size classes as one sequence: Flash-Next-like shapes, 4-bit gate/up, 6-bit down on "
                       "layers l % 4 == 0, 128 of 512 slots per layer (25%), 4096-token prefill chunk (passes of 64 "
                       "active experts, installs between passes), then 256 decode steps with L = 0.15"),
}


def build_streamer(cfg, seed, device, bits=None, max_tokens=None, n_shared=0, stream=None):
    import numpy as np
    import torch

    from streamed_quantized_expert_b200 import ops, synth
    from streamed_quantized_expert_b200.runtime import LayerSpec, Streamer, quantize_bank_gpu

    n_layers, E, k, H, I, g, bg, bd, T, S, _ = cfg
    descs = [ops.desc(E, k, H, I, g, *(bits(l) if bits else (bg, bd))) for l in range(n_layers)]
    banks = {}  # one layer's worth of distinct experts per size class, pinned
    for d in descs:
        if (d.bits_gu, d.bits_down) not in banks:
            banks[(d.bits_gu, d.bits_down)] = quantize_bank_gpu(E, d, seed + 17 * d.bits_down, device)
    # shared experts: the bank's last n_shared rows (distinct weights from a seed of their own)
    shared = {c: quantize_bank_gpu(n_shared, descs[0] if c is None else c, seed + 7919, device)
              for c in ([None] if n_shared else [])}
    specs = [LayerSpec(d, banks[(d.bits_gu, d.bits_down)], synth.bank_permutation(seed, l, E).tolist(),
                       shared[None] if n_shared else None)
             for l, d in enumerate(descs)]
    st = Streamer(specs, S, max_tokens=max_tokens or T, device=device, n_shared=n_shared, stream=stream)
    for l in range(n_layers):  # the S most popular experts start resident, on a random slot permutation
        hot = np.argsort(synth.popularity_rank(seed, l, E))[:S]
        st.place(l, hot.tolist(), synth.slot_permutation(seed, l, S).tolist())
    torch.cuda.synchronize(device)
    return st


def make_inputs(cfg, seed, n_steps, device, pinned=False, step0=0):
    import numpy as np
    import torch

    from streamed_quantized_expert_b200 import synth

    n_layers, E, k, H, I, g, bg, bd, T, S, _ = cfg
    xs = np.stack([np.stack([synth.activations(seed, l, T, H, step=step0 + s) for l in range(n_layers)])
                   for s in range(n_steps)])
    lg = np.stack([np.stack([synth.router_logits(seed, l, T, E, step=step0 + s) for l in range(n_layers)])
                   for s in range(n_steps)])
    x = torch.from_numpy(xs.view(np.int16))
    logits = torch.from_numpy(lg)
    if pinned:
        return x.pin_memory(), logits.pin_memory()
    return x.to(device), logits.to(device)


def ffn_graph_time(st, cfg, snaps, reps, device, T=None):
    """Time the FFN alone: a CUDA graph of the 48 layers' moe_expert_ffn calls
    (each with its layer's routing from one decode step of T tokens, default
    the configuration's), replayed `reps` times; returns microseconds per layer."""
    import torch

    from streamed_quantized_expert_b200 import ops

    n_layers, E, k, H, I, g, bg, bd, T0, S, _ = cfg
    T = T0 if T is None else T
    y = torch.zeros((T, H), dtype=torch.float32, device=device)
    g_ = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)
    with torch.cuda.graph(g_, stream=cap):
        cs = torch.cuda.current_stream(device)
        for l in range(n_layers):
            sn = snaps[l]
            ops.moe_expert_ffn(sn["x"], T, st.wdesc[l], st.pool_of(l), st.n_slots_of(l), st.table_dev[l],
                               sn["ids"], sn["w"], sn["offsets"], sn["pairs"], sn["meta"][2:], sn["meta"][0:1],
                               sn.get("xs"), 0, st.Ew, y, st.ws, st.ws_bytes, st.dev_err, cs)
    for _ in range(3):
        g_.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s = torch.cuda.current_stream(device)
    e0.record(s)
    for _ in range(reps):
        g_.replay()
    e1.record(s)
    torch.cuda.synchronize(device)
    us = 1e3 * e0.elapsed_time(e1) / (reps * n_layers)
    del g_
    return us


def stage_graph_times(st, cfg, snaps, logits, Lsub, reps, device):
    """Microseconds per call of route, sort and slot lookup: for each stage a
    CUDA graph of the layers' calls (each layer's own inputs from one decode
    step), replayed `reps` times, CUDA events."""
    import torch

    from streamed_quantized_expert_b200 import ops

    n_layers, _, _, H, I, g, bg, bd, T, S, _ = cfg
    E, k = st.Ew, st.kw  # the widened layer (shared experts after the routed ones)
    ids = torch.empty((T, k), dtype=torch.int32, device=device)
    w = torch.empty((T, k), dtype=torch.float32, device=device)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=device)
    pairs = torch.empty(max(T * k, 1), dtype=torch.int32, device=device)
    meta = torch.zeros(2 + 2 * E, dtype=torch.int32, device=device)
    slots = torch.empty(E, dtype=torch.int32, device=device)

    def route(l, cs):
        if st.ns:
            ops.moe_route_shared(logits[l], T, st.layers[l].desc, Lsub, st.table_dev[l], st.ns, None, ids, w, cs)
        else:
            ops.moe_route(logits[l], T, st.layers[l].desc, Lsub, st.table_dev[l], ids, w, cs)

    def sort(l, cs):
        sn = snaps[l]
        ops.moe_sort(sn["ids"], None, T, st.wdesc[l], offsets, pairs, meta[2:2 + E], meta[0:1], None, st.ws,
                     st.ws_bytes, cs)

    def lookup(l, cs):
        sn = snaps[l]
        ops.moe_slot_lookup(st.table_dev[l], sn["meta"][2:2 + E], sn["meta"][0:1], 0, E, st.n_slots_of(l), slots,
                            meta[2 + E:], meta[1:2], st.dev_err, cs)

    def route_sort_lookup(l, cs):  # the three in one launch (one token, no shared experts)
        ops.moe_route_sort_lookup(logits[l], T, st.layers[l].desc, Lsub, st.table_dev[l], st.n_slots_of(l), ids, w,
                                  offsets, pairs, meta[2:2 + E], meta[0:1], slots, meta[2 + E:], meta[1:2],
                                  st.dev_err, cs)

    out = {}
    stages = [("route", route), ("sort", sort), ("lookup", lookup)]
    if T == 1 and not st.ns:
        stages.append(("route_sort_lookup", route_sort_lookup))
    for name, fn in stages:
        g_ = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device)
        torch.cuda.synchronize(device)
        with torch.cuda.graph(g_, stream=cap):
            cs = torch.cuda.current_stream(device)
            for l in range(n_layers):
                fn(l, cs)
        for _ in range(3):
            g_.replay()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s_ = torch.cuda.current_stream(device)
        e0.record(s_)
        for _ in range(reps):
            g_.replay()
        e1.record(s_)
        torch.cuda.synchronize(device)
        out[name + "_us"] = round(1e3 * e0.elapsed_time(e1) / (reps * n_layers), 2)
        del g_
    out["how"] = ("per stage, a CUDA graph of the %d layers' calls (one decode step's inputs), replayed %d times, "
                  "CUDA events; route_sort_lookup: the three stages of one token in one launch, as the decode "
                  "driver runs them" % (n_layers, reps))
    return out


def run_prefill(args, rank, world, local_rank, name=None, layers=0, embedded=False):
    """Prefill chunk through every layer: route + sort (with sorted x), then
    passes of 64 active experts on the tensor-core grouped GEMM.  `value` is
    the expert FFN's TFLOP/s from a CUDA graph of every pass of every layer.
    embedded: the `prefill` object of another configuration's line (no e2e or
    oracle legs)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from streamed_quantized_expert_b200 import build as libbuild
    from streamed_quantized_expert_b200 import ops, synth
    from streamed_quantized_expert_b200.runtime import PASS_EXPERTS, LayerSpec, Streamer, quantize_bank_gpu

    libbuild.build()
    ops.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    n_layers, E, k, H, I, g, bits, T, desc_txt = PREFILL[name or args.config]
    layers = layers or args.layers
    if layers:
        n_layers = layers
        desc_txt += f" [{n_layers} of the layers]"
    seed = 1000 * rank
    descs = [ops.desc(E, k, H, I, g, *bits(l)) for l in range(n_layers)]
    banks = {}
    for d in descs:
        key = (d.bits_gu, d.bits_down)
        if key not in banks:
            banks[key] = quantize_bank_gpu(E, d, seed + 17 * d.bits_down, device)
    specs = [LayerSpec(d, banks[(d.bits_gu, d.bits_down)], synth.bank_permutation(seed, l, E).tolist())
             for l, d in enumerate(descs)]
    st = Streamer(specs, E, max_tokens=T, device=device)
    for l in range(n_layers):
        st.place(l, list(range(E)), synth.slot_permutation(seed, l, E).tolist())
    assert all(ops.moe_ffn_kernel_path(d, T, True) == ops.MOE_PATH_TC_PREFILL for d in descs)
    xs = torch.from_numpy(np.stack([synth.activations(seed, l, T, H).view(np.int16) for l in range(n_layers)]))
    lg = torch.from_numpy(np.stack([synth.router_logits(seed, l, T, E) for l in range(n_layers)]))
    x_d, lg_d = xs.to(device), lg.to(device)
    s = st.stream
    y = torch.zeros((T, H), dtype=torch.float32, device=device)

    # whole path (route, sort with sorted x, per pass: FFN), host-driven passes
    def whole(i0=0):
        for l in range(n_layers):
            st.prefill_layer(l, x_d[l], lg_d[l], T, y)

    for _ in range(args.warmup):
        whole()
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        whole()
    e1.record(s)
    torch.cuda.synchronize(device)
    whole_ms = e0.elapsed_time(e1) / args.steps

    # per-layer routing snapshots, then a CUDA graph of every pass of every layer
    snaps, n_act = [], []
    for l in range(n_layers):
        st.route_sort(l, x_d[l], lg_d[l], T, 0.0, want_sorted_x=True)
        torch.cuda.synchronize(device)
        snaps.append({"ids": st.ids[:T].clone(), "w": st.w[:T].clone(), "offsets": st.offsets.clone(),
                      "pairs": st.pairs[:T * k].clone(), "meta": st.meta.clone(),
                      "xs": st.x_sorted[:T * k].clone()})
        n_act.append(int(snaps[-1]["meta"][0].item()))
    g_ = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    with torch.cuda.graph(g_, stream=cap):
        cs = torch.cuda.current_stream(device)
        for l in range(n_layers):
            sn = snaps[l]
            y.zero_()
            for p in range(0, n_act[l], PASS_EXPERTS):
                ops.moe_expert_ffn(x_d[l], T, descs[l], st.pool_of(l), st.n_slots_of(l), st.table_dev[l],
                                   sn["ids"], sn["w"], sn["offsets"], sn["pairs"], sn["meta"][2:], sn["meta"][0:1],
                                   sn["xs"], p, PASS_EXPERTS, y, st.ws, st.ws_bytes, st.dev_err, cs)
    for _ in range(3):
        g_.replay()
    torch.cuda.synchronize(device)
    with ClockSampler(local_rank) as clk:
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        for _ in range(args.ffn_reps):
            g_.replay()
        f1.record(s)
        torch.cuda.synchronize(device)
    ffn_ms = f0.elapsed_time(f1) / args.ffn_reps  # all layers
    del g_
    ffn_ms, whole_ms = max_over_ranks([ffn_ms, whole_ms], device)
    err = st.check_dev_err()
    hbm_peak, tf_peak, peak_kind = peaks()
    flops = sum(2.0 * T * k * 3 * H * I for _ in range(n_layers))
    slot_b = [ops.moe_slot_bytes(d) for d in descs]
    bytes_ = sum(n_act[l] * slot_b[l] + T * H * 2 + T * H * 4 for l in range(n_layers))
    tflops = flops / (ffn_ms * 1e-3) / 1e12
    gbs = bytes_ / (ffn_ms * 1e-3) / 1e9
    ffn_obj = {"ms_all_layers": round(ffn_ms, 3), "us_per_layer": round(1e3 * ffn_ms / n_layers, 1),
               "tflops": round(tflops, 2), "hbm_gbs": round(gbs, 1),
               "tok_s_equiv": round(T / (ffn_ms * 1e-3), 1),
               "how": "CUDA graph of every pass (moe_expert_ffn) of every layer, replayed %d times, CUDA events"
                      % args.ffn_reps}
    roof = {"bound": "tensor", "achieved": round(tflops, 2), "peak": tf_peak, "unit": "TFLOP/s",
            "frac": round(tflops / tf_peak, 4),
            # the capture covers the 1024-token Flash-Next-like chunk only
            "traffic": recorded_traffic("pf_gemm_kernel") if (name or args.config) == "prefill" else None,
            "traffic_note": "DRAM bytes of one 64-expert pass's gate/up + down launches of the 1024-token "
                            "Flash-Next-like chunk (profiles/traffic.txt); null for other workloads",
            "hbm": {"achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s", "frac": round(gbs / hbm_peak, 4)},
            "kernel": "pf_gemm_kernel (gate/up + SwiGLU, down) + combine, per pass",
            "flops_per_layer": 2.0 * T * k * 3 * H * I, "peak_kind": peak_kind}
    if embedded:
        del st
        torch.cuda.empty_cache()
        return {"workload": desc_txt, "value": round(tflops, 2), "unit": "TFLOP/s", "tokens": T, "layers": n_layers,
                "active_experts_per_layer": round(sum(n_act) / n_layers, 1),
                "ms_per_chunk_whole_path": round(whole_ms, 3), "ffn": ffn_obj, "roofline": roof,
                "l2": "inputs larger than L2: %.0f MB of expert slots per replay" % (bytes_ / 1e6),
                "gpu_launches_per_replay": sum((n_act[l] + PASS_EXPERTS - 1) // PASS_EXPERTS
                                               for l in range(n_layers)) * 3}

    # e2e: x and logits from pinned host memory, y of every layer read back
    xh, lgh = xs.pin_memory(), lg.pin_memory()
    yh = torch.empty((n_layers, T, H), dtype=torch.float32).pin_memory()
    xd2 = torch.empty_like(x_d)
    lgd2 = torch.empty_like(lg_d)
    torch.cuda.synchronize(device)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(s)
    for _ in range(args.steps):
        with torch.cuda.stream(s):
            xd2.copy_(xh, non_blocking=True)
            lgd2.copy_(lgh, non_blocking=True)
        for l in range(n_layers):
            st.prefill_layer(l, xd2[l], lgd2[l], T, y)
            with torch.cuda.stream(s):
                yh[l].copy_(y, non_blocking=True)
    h1.record(s)
    torch.cuda.synchronize(device)
    e2e_ms = h0.elapsed_time(h1) / args.steps
    if rank != 0:
        return None
    return {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "value_is": "prefill expert-FFN TFLOP/s over every pass of %d layers (CUDA graph)" % n_layers,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(whole_ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp16 tensor-core operands (weights dequantised from 3/4/6-bit codes, or bf16 weights converted; "
                 "x and h in fp16), fp32 TMEM accumulate",
        "data": "synthetic (seeded N(0,0.02) experts quantised on the GPU; N(0,1) bf16 x; log-Zipf-biased logits)",
        "config": {"workload": desc_txt, "layers": n_layers, "experts": E, "top_k": k, "hidden": H,
                   "intermediate": I, "group": g, "tokens": T,
                   "bits_per_layer": sorted({tuple(bits(l)) for l in range(n_layers)}),
                   "active_experts_per_layer": round(sum(n_act) / n_layers, 1),
                   "l2": "inputs larger than L2: %.0f MB of expert slots per replay" % (bytes_ / 1e6),
                   "parallelism": f"replicas x{world} (independent chunks)"},
        "ffn": ffn_obj,
        "whole_path": {"ms_per_chunk": round(whole_ms, 3), "tok_s": round(T / (whole_ms * 1e-3), 1),
                       "how": "route + sort (sorted x) + host-driven passes of the FFN, every layer"},
        "roofline": roof,
        "gpu_launches": sum((n_act[l] + PASS_EXPERTS - 1) // PASS_EXPERTS for l in range(n_layers)) * 3 * args.ffn_reps,
        "dev_err": err,
        "clocks": clk.summary(),
        "e2e": {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "tok_s": round(T / (e2e_ms * 1e-3), 1),
                "h2d_bytes_per_step": int(xs.numel() * 2 + lg.numel() * 4),
                "d2h_bytes_per_step": int(n_layers * T * H * 4)},
        **({} if args.no_cpu_baseline else {"cpu_baseline": cpu_baseline_prefill(PREFILL[args.config], seed)}),
    }


def run_sequence(args, rank, world, local_rank):
    """Prefill chunk, then decode steps, on one cache (see SEQUENCE).  `value`
    is the decode tok/s of the whole path after the prefill; the prefill
    chunk's time (with its installs) and both phases' miss rates are reported,
    and the same sequence is replayed from the same initial cache with L = 0
    (untimed) for the miss rate without substitution."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from streamed_quantized_expert_b200 import build as libbuild
    from streamed_quantized_expert_b200 import ops, synth

    libbuild.build()
    ops.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    n_layers, E, k, H, I, g, bits, Tp, n_dec, S, Lsub, desc_txt = SEQUENCE[args.config]
    if args.layers:
        n_layers = args.layers
        desc_txt += f" [{n_layers} of the layers]"
    n_dec = args.decode_steps or n_dec
    seed = 1000 * rank
    cfg = (n_layers, E, k, H, I, g, 4, 4, 1, S, desc_txt)
    # prefill inputs (x of four distinct layers reused: the FFN's work does not depend on it), decode inputs
    xs_p = [torch.from_numpy(synth.activations(seed, l, Tp, H).view(np.int16)).to(device) for l in range(4)]
    lg_p = [torch.from_numpy(synth.router_logits(seed, l, Tp, E)).to(device) for l in range(n_layers)]
    x_d, lg_d = make_inputs(cfg, seed, n_dec, device, step0=1)
    y = torch.zeros((Tp, H), dtype=torch.float32, device=device)

    def sequence(st, L):
        s = st.stream
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        i0 = st.installs
        ev[0].record(s)
        for l in range(n_layers):
            st.prefill_layer(l, xs_p[l % 4], lg_p[l], Tp, y)
        ev[1].record(s)
        i1 = st.installs
        ev[2].record(s)
        for i in range(n_dec):
            for l in range(n_layers):
                st.decode_layer(l, x_d[i, l], lg_d[i, l], 1, L)
        ev[3].record(s)
        torch.cuda.synchronize(device)
        return (ev[0].elapsed_time(ev[1]), ev[2].elapsed_time(ev[3]), i1 - i0, st.installs - i1,
                st.installed_bytes)

    st = build_streamer(cfg, seed, device, bits, max_tokens=Tp)
    if world > 1:
        dist.barrier()
    with ClockSampler(local_rank) as clk:
        pf_ms, dec_ms, pf_inst, dec_inst, inst_bytes = sequence(st, Lsub)
    pf_ms, dec_ms = max_over_ranks([pf_ms, dec_ms], device)
    err = st.check_dev_err()
    del st
    torch.cuda.empty_cache()
    st0 = build_streamer(cfg, seed, device, bits, max_tokens=Tp)
    _, _, pf_inst0, dec_inst0, _ = sequence(st0, 0.0)
    del st0
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    flops = 2.0 * Tp * k * 3 * H * I * n_layers
    pairs_pf = Tp * k * n_layers
    pairs_dec = n_dec * k * n_layers
    return {
        "metric": METRIC, "value": round(n_dec * world / (dec_ms * 1e-3), 3), "unit": "tok/s",
        "value_is": "decode tok/s of the whole path (route+sort+lookup+installs+FFN+combine, %d layers) after the "
                    "prefill chunk, from the cache it left" % n_layers,
        "n_gpus": world, "steps": n_dec, "warmup": 0, "ms_per_step": round(dec_ms / n_dec, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 (4/6-bit codes, bf16 tensor-core operands, fp32 accumulate)",
        "data": "synthetic (seeded N(0,0.02) experts quantised on the GPU; N(0,1) bf16 x; log-Zipf-biased logits)",
        "config": {"workload": desc_txt, "layers": n_layers, "experts": E, "top_k": k, "hidden": H, "intermediate": I,
                   "group": g, "prefill_tokens": Tp, "decode_steps": n_dec, "slots_per_layer": S,
                   "substitution_L": Lsub, "parallelism": f"replicas x{world}"},
        "prefill": {"ms_per_chunk": round(pf_ms, 3), "tok_s": round(Tp / (pf_ms * 1e-3), 1),
                    "tflops_with_installs": round(flops / (pf_ms * 1e-3) / 1e12, 2),
                    "installs": pf_inst, "miss_rate": round(pf_inst / pairs_pf, 5),
                    "how": "route + sort + per pass of 64 active experts: lookup, host LRU step, pinned installs, "
                           "FFN (host-driven passes), every layer, CUDA events"},
        "decode": {"ms_per_token": round(dec_ms / n_dec, 4), "installs": dec_inst,
                   "miss_rate": round(dec_inst / pairs_dec, 4),
                   "miss_rate_without_substitution": round(dec_inst0 / pairs_dec, 4),
                   "prefill_installs_without_substitution": pf_inst0},
        "dev_err": err, "clocks": clk.summary(),
    }


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from streamed_quantized_expert_b200 import build as libbuild
    from streamed_quantized_expert_b200 import ops

    libbuild.build()
    ops.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    cfg = CONFIGS[args.config]
    n_layers, E, k, H, I, g, bg, bd, T, S, desc_txt = cfg
    extra = DECODE_EXTRA.get(args.config, {})
    Lsub = extra.get("L", 0.0)
    seed = 1000 * rank
    # a step captured as a CUDA graph runs on a stream of its own (capture needs a non-default stream)
    st = build_streamer(cfg, seed, device, extra.get("bits"), n_shared=extra.get("n_shared", 0),
                        stream=torch.cuda.Stream(device) if extra.get("graph_step") else None)
    steps_total = args.warmup + args.steps
    # the popularity bias of the logits and the initially resident experts come from the same seed
    x, logits = make_inputs(cfg, seed, steps_total + 1, device)
    s = st.stream

    def step(i, x_src, lg_src):
        for l in range(n_layers):
            st.decode_layer(l, x_src[i, l], lg_src[i, l], T, Lsub)

    for i in range(args.warmup):
        step(i, x, logits)
    torch.cuda.synchronize(device)
    graphs = []
    if extra.get("graph_step"):
        # every layer fully resident: the driver never waits on the host, so each
        # timed step (its own inputs) is captured once and replayed in the timed region
        if any(st.cache.resident(l) < E for l in range(n_layers)):
            raise RuntimeError("graph_step needs every expert of every layer resident")
        l_cap = st.launches
        for i in range(args.warmup, steps_total):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=s):
                step(i, x, logits)
            graphs.append(gr)
        torch.cuda.synchronize(device)
        graph_launches = (st.launches - l_cap) // max(len(graphs), 1)
    if world > 1:
        dist.barrier()

    inst0, bytes0, l0 = st.installs, st.installed_bytes, st.launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize(device)
        e0.record(s)
        for i in range(args.warmup, steps_total):
            if graphs:
                with torch.cuda.stream(s):  # replayed on the stream the events are recorded on
                    graphs[i - args.warmup].replay()
            else:
                step(i, x, logits)
        e1.record(s)
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1)
        launches = st.launches - l0 if not graphs else graph_launches * len(graphs)
        installs, inst_bytes = st.installs - inst0, st.installed_bytes - bytes0
        del graphs

        # one more (untimed) step whose per-layer routing is kept for the FFN-only replay
        snaps = []
        for l in range(n_layers):
            st.decode_layer(l, x[steps_total, l], logits[steps_total, l], T, Lsub)
            snaps.append({"x": x[steps_total, l], "ids": st.ids.clone(), "w": st.w.clone(),
                          "offsets": st.offsets.clone(), "pairs": st.pairs.clone(), "meta": st.meta.clone(),
                          **({"xs": st.x_sorted[:T * st.kw].clone()} if st.uses_tc(l, T) else {})})
        torch.cuda.synchronize(device)
        n_unique = sum(int(sn["meta"][0].item()) for sn in snaps) / n_layers
        ffn_us = ffn_graph_time(st, cfg, snaps, args.ffn_reps, device)
        stage_us = stage_graph_times(st, cfg, snaps, logits[steps_total], Lsub, args.ffn_reps, device)
        # batch sweep (configurations that name one): the same step's first T2 tokens through every layer
        sweep = []
        for T2 in SWEEP.get(args.config, ()):
            sn2 = []
            for l in range(n_layers):
                st.decode_layer(l, x[steps_total, l, :T2], logits[steps_total, l, :T2], T2, Lsub)
                sn2.append({"x": x[steps_total, l, :T2], "ids": st.ids.clone(), "w": st.w.clone(),
                            "offsets": st.offsets.clone(), "pairs": st.pairs.clone(), "meta": st.meta.clone(),
                            **({"xs": st.x_sorted[:T2 * st.kw].clone()} if st.uses_tc(l, T2) else {})})
            torch.cuda.synchronize(device)
            us2 = ffn_graph_time(st, cfg, sn2, args.ffn_reps, device, T=T2)
            sweep.append((T2, us2, sn2))
    ms_max = max_over_ranks([ms], device)[0]
    err = st.check_dev_err()
    miss_no_sub = None
    if Lsub > 0:  # the same token sequence from the same initial cache, without substitution (untimed)
        st0 = build_streamer(cfg, seed, device, extra.get("bits"))
        base0 = 0
        for i in range(steps_total):
            if i == args.warmup:
                base0 = st0.installs
            for l in range(n_layers):
                st0.decode_layer(l, x[i, l], logits[i, l], T, 0.0)
        torch.cuda.synchronize(device)
        miss_no_sub = round((st0.installs - base0) / max(args.steps * n_layers * T * k, 1), 4)
        del st0
        torch.cuda.empty_cache()

    # e2e: inputs from pinned host memory copied in, y of every layer read back, same K steps
    # (each step: one copy in of every layer's x and logits, one copy back of every layer's y)
    xh, lgh = make_inputs(cfg, seed, args.steps, device, pinned=True, step0=steps_total + 1)
    yh = torch.empty((args.steps, n_layers, T, H), dtype=torch.float32).pin_memory()
    xd = torch.empty((n_layers, T, H), dtype=torch.int16, device=device)
    lgd = torch.empty((n_layers, T, E), dtype=torch.float32, device=device)
    yd = torch.empty((n_layers, T, H), dtype=torch.float32, device=device)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s)
    for i in range(args.steps):
        with torch.cuda.stream(s):
            xd.copy_(xh[i], non_blocking=True)
            lgd.copy_(lgh[i], non_blocking=True)
        for l in range(n_layers):
            st.decode_layer(l, xd[l], lgd[l], T, Lsub, y=yd[l])
        with torch.cuda.stream(s):
            yh[i].copy_(yd, non_blocking=True)
    f1.record(s)
    torch.cuda.synchronize(device)
    e2e_ms = f0.elapsed_time(f1)
    e2e_ms_max = max_over_ranks([e2e_ms], device)[0]
    copy_gbs = install_copy_rate(st, device)
    prefill_obj = None
    if args.config == "decode" and args.prefill_layers > 0:
        prefill_obj = run_prefill(args, rank, world, local_rank, name="prefill", layers=args.prefill_layers,
                                  embedded=True)

    if rank != 0:
        return None
    hbm_peak, tf_peak, peak_kind = peaks()
    tokens = args.steps * T * world
    from streamed_quantized_expert_b200 import ops as _ops

    slot_bytes = [_ops.moe_slot_bytes(st.layers[l].desc) for l in range(n_layers)]
    ffn_bytes = (sum(int(sn["meta"][0].item()) * slot_bytes[l] for l, sn in enumerate(snaps)) / n_layers
                 + T * H * 2 + T * H * 4)
    achieved = ffn_bytes / (ffn_us * 1e-6) / 1e9
    flops_per_ffn = 2.0 * T * k * 3 * H * I
    out = {
        "metric": METRIC,
        "value": round(tokens / (ms_max / 1e3), 3),
        "unit": "tok/s",
        "value_is": ("decode tok/s of the whole path (route+sort+FFN+combine, %d layers, every expert resident: one "
                     "CUDA graph per step, replayed)" if extra.get("graph_step") else
                     "decode tok/s of the whole path (route+sort+lookup+installs+FFN+combine, %d layers)") % n_layers,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 (3/4/6-bit codes, bf16 tensor-core operands, fp32 accumulate)",
        "data": "synthetic (seeded N(0,0.02) experts quantised on the GPU; N(0,1) bf16 x; log-Zipf-biased logits)",
        "config": {"workload": desc_txt, "layers": n_layers, "experts": E, "top_k": k, "hidden": H,
                   "intermediate": I, "group": g, "bits": [bg, bd], "tokens_per_step": T, "slots_per_layer": S,
                   "l2": "inputs larger than L2: each step reads ~%.0f MB of distinct expert slots" %
                         (n_layers * ffn_bytes / 1e6),
                   "parallelism": f"replicas x{world} (independent token streams)",
                   **({"shared_experts": st.ns} if st.ns else {})},
        "ffn": {"tok_s_equiv": round(T / (n_layers * ffn_us * 1e-6), 1),
                "us_per_layer": round(ffn_us, 3),
                "hbm_gbs": round(achieved, 1),
                "tflops": round(flops_per_ffn / (ffn_us * 1e-6) / 1e12, 3),
                "how": "CUDA graph of the %d layers' moe_expert_ffn calls, replayed %d times, CUDA events" %
                       (n_layers, args.ffn_reps)},
        "stages": stage_us,
        "installs": {"experts": installs, "per_token": round(installs / max(args.steps * T, 1), 2),
                     "gbs": round(inst_bytes / (ms * 1e-3) / 1e9, 2),
                     "gbs_is": "installed bytes / timed region (the share of the host link the steps use)",
                     "copy_gbs": copy_gbs,
                     "copy_gbs_is": "moe_install_slots of 32 experts from pinned host alone, CUDA events on the side "
                                    "stream (the host-to-device rate an install gets)",
                     "miss_rate": round(installs / max(args.steps * n_layers * T * k, 1), 4),
                     "bytes": inst_bytes, "substitution_L": Lsub,
                     **({} if miss_no_sub is None else
                        {"miss_rate_without_substitution": miss_no_sub,
                         "how_compared": "same tokens and initial cache, L = 0, installs of the timed steps"})},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4),
                     # the capture covers the default decode workload only
                     "traffic": recorded_traffic("ffn_fused_kernel") if args.config == "decode" else None,
                     "kernel": ("ffn_fused_kernel (one launch per layer: every CTA gate/up + SwiGLU items, then the "
                                "first H/16 CTAs a down + combine tile, over launch-tagged h words)" if T <= 8 and T * k <= 64 else
                                "pf_gemm_kernel (tcgen05 grouped GEMM: gate/up + SwiGLU, down) + combine, per layer"
                                if st.uses_tc(0, T) else
                                "moe_expert_ffn (gate/up+SwiGLU kernel + down kernel), per layer"),
                     "bytes_per_launch": int(ffn_bytes), "peak_kind": peak_kind},
        **({"batch_sweep": [
            {"tokens": T2, "us_per_layer": round(us2, 2),
             "hbm_gbs": round(b2 / (us2 * 1e-6) / 1e9, 1), "frac": round(b2 / (us2 * 1e-6) / 1e9 / hbm_peak, 4),
             "unique_experts_per_layer": round(nu2, 1),
             "kernel_path": ["fused decode", "GEMV", "tcgen05 grouped GEMM"][
                 _ops.moe_ffn_kernel_path(st.layers[0].desc, T2, st.uses_tc(0, T2))]}
            for T2, us2, nu2, b2 in [
                (T2, us2, sum(int(sn["meta"][0].item()) for sn in sn2) / n_layers,
                 sum(int(sn["meta"][0].item()) * slot_bytes[l] for l, sn in enumerate(sn2)) / n_layers
                 + T2 * H * 6)
                for T2, us2, sn2 in sweep + [(T, ffn_us, snaps)]]]} if sweep else {}),
        "gpu_launches": launches,
        "dev_err": err,
        "clocks": clk.summary(),
        "e2e": {"value": round(tokens / (e2e_ms_max / 1e3), 3), "unit": "tok/s",
                "h2d_bytes_per_step": n_layers * (T * H * 2 + T * E * 4),
                "d2h_bytes_per_step": n_layers * T * H * 4},
    }
    if prefill_obj is not None:
        out["prefill"] = prefill_obj
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, seed, samples=args.cpu_layers)
    return out


# Guessed prefetch: hidden states as a residual stream, per-layer routers on
# the GPU (moe_router_logits), the next two layers' routers evaluated on each
# layer's state, their guessed misses read ahead (moe_decode_layer_ahead).
# name: (layers, E, k, H, I, g, bits_gu, bits_down, T, slots per layer, description)
AHEAD = {
    "decode_ahead": (48, 512, 10, 2048, 512, 64, 3, 3, 1, 192,
                     "Flash-Next-like decode with guessed prefetch: 48 layers x 512 experts, top-10, H 2048, I 512, "
                     "3-bit g64, 1 token/step, 192 slots/layer, misses installed from pinned host; hidden states a "
                     "residual stream (consecutive layers at correlation 0.89), logits = router(x) on the GPU, the "
                     "next two layers' routers run on each layer's state and their guessed misses read ahead"),
}


def run_decode_ahead(args, rank, world, local_rank):
    """The same token sequence twice from the same initial cache: plain
    decode layers, then decode layers with guessed prefetch; both time the
    whole path including the routers."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from streamed_quantized_expert_b200 import build as libbuild
    from streamed_quantized_expert_b200 import ops, synth

    libbuild.build()
    ops.lib()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    cfg = AHEAD[args.config]
    n_layers, E, k, H, I, g, bg, bd, T, S, desc_txt = cfg
    seed = 1000 * rank
    steps_total = args.warmup + args.steps
    xs = torch.from_numpy(np.stack([synth.hidden_stream(seed, n_layers, T, H, step=i)
                                    for i in range(steps_total)]).view(np.int16)).to(device)
    Wr = torch.from_numpy(np.stack([synth.router_weights(seed, l, E, H) for l in range(n_layers)]).view(np.int16)
                          ).to(device)
    br = torch.from_numpy(np.stack([synth.router_bias(seed, l, E) for l in range(n_layers)])).to(device)
    scale = 1.0 / float(np.sqrt(H))
    logits = torch.empty((n_layers, T, E), dtype=torch.float32, device=device)
    glog = torch.empty((n_layers, 2, T, E), dtype=torch.float32, device=device)
    results = {}
    for mode in ("plain", "ahead"):
        st = build_streamer(cfg, seed, device)
        s = st.stream

        def step(i):
            for l in range(n_layers):
                ops.moe_router_logits(xs[i, l], T, Wr[l], br[l], scale, E, H, logits[l], s)
                if mode == "plain":
                    st.decode_layer(l, xs[i, l], logits[l], T, 0.0)
                    continue
                guesses = []
                for d in range(1, args.ahead_layers + 1):
                    if l + d < n_layers:
                        ops.moe_router_logits(xs[i, l], T, Wr[l + d], br[l + d], scale, E, H, glog[l, d - 1], s)
                        guesses.append((l + d, glog[l, d - 1], args.ahead_top))
                st.decode_layer_ahead(l, xs[i, l], logits[l], T, 0.0, guesses)

        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
        inst0, bytes0, pf0 = st.installs, st.installed_bytes, st.prefetch.stats()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank) as clk:
            torch.cuda.synchronize(device)
            e0.record(s)
            for i in range(args.warmup, steps_total):
                step(i)
            e1.record(s)
            torch.cuda.synchronize(device)
        st.ahead.synchronize()
        ms = max_over_ranks([e0.elapsed_time(e1)], device)[0]
        pf = {key: v - pf0[key] for key, v in st.prefetch.stats().items()}
        results[mode] = {"ms": ms, "installs": st.installs - inst0, "bytes": st.installed_bytes - bytes0, "pf": pf,
                         "clocks": clk.summary(), "dev_err": st.check_dev_err(), "launches": st.launches}
        del st
        torch.cuda.empty_cache()
    if rank != 0:
        return None
    r0, r1 = results["plain"], results["ahead"]
    tokens = args.steps * T * world
    sb = ops.moe_slot_bytes(ops.desc(E, k, H, I, g, bg, bd))
    pf = r1["pf"]
    per_tok = lambda v: round(v / max(args.steps * T, 1), 2)
    return {
        "metric": METRIC,
        "value": round(tokens / (r1["ms"] / 1e3), 3),
        "unit": "tok/s",
        "value_is": "decode tok/s of the whole path with guessed prefetch (routers + route+sort+lookup+installs+FFN"
                    "+combine, %d layers)" % n_layers,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(r1["ms"] / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 (3-bit codes, bf16 tensor-core operands, fp32 accumulate)",
        "data": "synthetic (seeded N(0,0.02) experts quantised on the GPU; residual-stream bf16 hidden states; "
                "N(0,1) bf16 routers with a log-Zipf popularity bias)",
        "config": {"workload": desc_txt, "layers": n_layers, "experts": E, "top_k": k, "hidden": H,
                   "intermediate": I, "group": g, "bits": [bg, bd], "tokens_per_step": T, "slots_per_layer": S,
                   "guessed_layers_ahead": args.ahead_layers, "guesses_read_per_token": args.ahead_top or k,
                   "parallelism": f"replicas x{world} (independent token streams)"},
        "without_prefetch": {"value": round(tokens / (r0["ms"] / 1e3), 3), "unit": "tok/s",
                             "ms_per_step": round(r0["ms"] / args.steps, 4),
                             "installs_per_token": per_tok(r0["installs"])},
        "installs": {"per_token": per_tok(r1["installs"]),
                     "guessed_per_token": per_tok(pf["guessed"]),
                     "guessed_copies_per_token": per_tok(pf["started"]),
                     "guesses_entered_per_token": per_tok(pf["entered"]),
                     "guesses_wasted_per_token": per_tok(pf["wasted"]),
                     "skipped_in_flight_per_token": per_tok(pf["skipped_in_flight"]),
                     "bytes_per_token": round((r1["bytes"] + pf["started"] * sb) / max(args.steps * T, 1)),
                     "how": "installs: the layers' own misses; guessed: distinct experts of the two guessed "
                            "layers' top-k per layer; copies: guesses absent from the cache; entered: copies "
                            "that landed before their layer ran and found their expert still absent"},
        "dev_err": r0["dev_err"] | r1["dev_err"],
        "clocks": r1["clocks"],
    }


def install_copy_rate(st, device, n=32, reps=3):
    """GB/s of moe_install_slots copying n experts' slot bytes from the pinned
    bank into a scratch pool (best of `reps`), CUDA events on the side stream."""
    import torch

    from streamed_quantized_expert_b200 import ops

    sb = st.class_bytes[st.layer_class[0]]
    n = min(n, st.E)
    scratch = torch.empty(n * sb, dtype=torch.uint8, device=device)
    rows = [st._row_addr(0, e) for e in range(n)]
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st.side)
        ops.moe_install_slots(scratch, sb, n, rows, list(range(n)), st.side, None)
        e1.record(st.side)
        e1.synchronize()
        best = max(best, n * sb / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del scratch
    return round(best, 2)


# ---------------------------------------------------------------------------
# oracle (CPU) timing
# ---------------------------------------------------------------------------
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _oracle_bank(cfg, seed, rows=61):
    """`rows` distinct experts quantised by the oracle (expert e uses row e % rows),
    built on a thread pool: the experts' slot bytes are prepared outside any timing."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle as orc
    from streamed_quantized_expert_b200 import synth

    n_layers, E, k, H, I, g, bg, bd = cfg[:8]
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        return list(ex.map(lambda r: orc.build_slot(*synth.expert_weights(seed, r, H, I), g, bg, bd), range(rows)))


def _oracle_layer(cfg, seed, l, bank, step=0):
    """Inputs of one decode layer for the oracle: x, logits, slots, table."""
    import numpy as np

    from streamed_quantized_expert_b200 import synth

    n_layers, E, k, H, I, g, bg, bd, T, S = cfg[:10]
    x = synth.activations(seed, l, T, H, step=step)
    logits = synth.router_logits(seed, l, T, E, step=step)
    slots = [bank[e % len(bank)] for e in range(E)]
    table = np.full(E, -1, np.int32)
    table[:S] = np.arange(S)
    return x, logits, slots, table


def _oracle_decode_layer(cfg, inp):
    """route + sort + lookup + FFN/combine of one decode layer by the oracle as it stands."""
    import oracle as orc

    n_layers, E, k, H, I, g, bg, bd, T, S = cfg[:10]
    x, logits, slots, table = inp
    ids, w, _ = orc.route(logits, k)
    off, pairs, active = orc.sort(ids, E)
    orc.slot_lookup(table, active, 0, E, S)
    orc.expert_ffn(x, H, I, g, bg, bd, ids, w, slots)


def _time_layers(cfg, inputs, threads):
    """Seconds to run the oracle on every layer of `inputs`, `threads` at a time
    (a thread pool: the oracle's C calls release the GIL)."""
    from concurrent.futures import ThreadPoolExecutor

    t0 = time.perf_counter()
    if threads <= 1:
        for inp in inputs:
            _oracle_decode_layer(cfg, inp)
    else:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda inp: _oracle_decode_layer(cfg, inp), inputs))
    return time.perf_counter() - t0


def cpu_baseline(cfg, seed, samples=8):
    """The oracle as it stands on a bounded sample: `samples` layers of one
    decode step (route, sort, lookup, FFN + combine), on all host cores (one
    layer per thread) and on one core; tok/s scaled to all layers."""
    n_layers, T = cfg[0], cfg[8]
    samples = max(1, min(samples, n_layers))
    bank = _oracle_bank(cfg, seed)
    inputs = [_oracle_layer(cfg, seed, l, bank) for l in range(samples)]
    cores = os.cpu_count() or 1
    threads = min(cores, samples)
    dt_all = _time_layers(cfg, inputs, threads)
    dt_one = _time_layers(cfg, inputs[:max(1, samples // 4)], 1) * samples / max(1, samples // 4)
    rate = lambda dt: T / (dt / samples * n_layers)
    return {"value": round(rate(dt_all), 6), "unit": "tok/s", "cores": threads, "kind": "oracle",
            "host_cores": cores, "cpu_model": cpu_model(),
            "single_core": {"value": round(rate(dt_one), 6), "cores": 1},
            "sample": f"{samples} of {n_layers} layers of one {T}-token decode step (route+sort+lookup+FFN), "
                      f"one layer per thread on {threads} threads ({dt_all:.2f} s), scaled to {n_layers} layers; "
                      f"single core timed on {max(1, samples // 4)} of the layers"}


def cpu_baseline_prefill(pcfg, seed, n_tok=6):
    """The oracle as it stands, single-threaded, on a bounded sample of a
    prefill chunk: route + sort of the whole chunk of layer 0, then the FFN of
    `n_tok` of its tokens (the oracle computes tokens one by one); the rate is
    the sample's FFN flops over its time."""
    import numpy as np

    import oracle as orc
    from streamed_quantized_expert_b200 import synth

    n_layers, E, k, H, I, g, bits, T, _ = pcfg
    bg, bd = bits(0)
    x = synth.activations(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    tok = np.linspace(0, T - 1, n_tok).astype(int)
    ids, _, _ = orc.route(logits[tok], k)
    slots = [None] * E
    for e in np.unique(ids):
        slots[int(e)] = orc.build_slot(*synth.expert_weights(seed, int(e), H, I), g, bg, bd)
    t0 = time.perf_counter()
    ids_all, w_all, _ = orc.route(logits, k)
    orc.sort(ids_all, E)
    ids_s, w_s, _ = orc.route(logits[tok], k)
    orc.expert_ffn(x[tok], H, I, g, bg, bd, ids_s, w_s, slots)
    dt = time.perf_counter() - t0
    flops = 2.0 * n_tok * k * 3 * H * I
    return {"value": round(flops / dt / 1e12, 9), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"layer 0: route + sort of the {T}-token chunk, FFN of {n_tok} sampled tokens "
                      f"({dt:.2f} s of CPU time)"}


def run_reference(args, rank):
    """The reference arm: the oracle as it stands on the host cores, with our
    arm's metric, unit and configuration.  Each step is a bounded sample of the
    workload (decode: one token through as many layers as there are cores, one
    layer per thread; prefill: the chunk's route + sort and the FFN of a few of
    its tokens); ms_per_step is the measured time of that sample."""
    if rank != 0:
        return None
    cores = os.cpu_count() or 1
    if args.config in PREFILL:
        pcfg = PREFILL[args.config]
        times, vals = [], []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            r = cpu_baseline_prefill(pcfg, 7 + i, n_tok=2)
            if i >= args.warmup:
                times.append(time.perf_counter() - t0)
                vals.append(r["value"])
        v = statistics.mean(vals)
        return {"metric": METRIC, "impl": "reference", "value": v, "unit": "TFLOP/s",
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 * statistics.mean(times), 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
                "data": "synthetic", "config": {"workload": pcfg[-1]},
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                                 "host_cores": cores, "cpu_model": cpu_model(),
                                 "sample": "per step: route + sort of layer 0's chunk, FFN of 2 sampled tokens"},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    cfg = CONFIGS[args.config]
    n_layers, E, k, H, I, g, bg, bd, T, S, desc_txt = cfg
    threads = max(1, min(cores, n_layers))
    bank = _oracle_bank(cfg, 7)
    times = []
    for i in range(args.warmup + args.steps):
        inputs = [_oracle_layer(cfg, 7, l, bank, step=i) for l in range(threads)]
        dt = _time_layers(cfg, inputs, threads)
        if i >= args.warmup:
            times.append(dt)
    t = statistics.mean(times)
    v = T / (t * n_layers / threads)
    sample = (f"per step: one {T}-token decode step through {threads} of the {n_layers} layers (route+sort+lookup+"
              f"FFN), one layer per thread; tok/s scaled to {n_layers} layers")
    return {"metric": METRIC, "impl": "reference", "value": v, "unit": "tok/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic", "config": {"workload": desc_txt},
            "cpu_baseline": {"value": v, "unit": "tok/s", "cores": threads, "kind": "oracle", "host_cores": cores,
                             "cpu_model": cpu_model(), "sample": sample},
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS) + sorted(PREFILL) + sorted(SEQUENCE) + sorted(AHEAD),
                    default="decode")
    ap.add_argument("--cpu-layers", type=int, default=8)
    ap.add_argument("--ahead-layers", type=int, default=2, help="decode_ahead: layers guessed ahead (0..2)")
    ap.add_argument("--ahead-top", type=int, default=0, help="decode_ahead: best guesses read per token (0 = k)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ffn-reps", type=int, default=20)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (small profiling runs)")
    ap.add_argument("--decode-steps", type=int, default=0, help="mixed_sequence: decode steps (default 256)")
    ap.add_argument("--prefill-layers", type=int, default=8,
                    help="decode line: layers of the Flash-Next-like prefill chunk timed into its `prefill` object "
                         "(0: none)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.layers and args.config in CONFIGS:
        c = list(CONFIGS[args.config])
        c[0] = args.layers
        c[-1] = c[-1] + f" [layers overridden to {args.layers}]"
        CONFIGS[args.config] = tuple(c)
    if args.impl == "reference":
        out = run_reference(args, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    import datetime

    import torch
    import torch.distributed as dist

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run = (run_prefill if args.config in PREFILL else run_sequence if args.config in SEQUENCE else
               run_decode_ahead if args.config in AHEAD else run_ours)
        out = run(args, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
