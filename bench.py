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
def build_streamer(cfg, seed, device):
    import numpy as np
    import torch

    from streamed_quantized_expert_b200 import ops, synth
    from streamed_quantized_expert_b200.runtime import LayerSpec, Streamer, quantize_bank_gpu

    n_layers, E, k, H, I, g, bg, bd, T, S, _ = cfg
    d = ops.desc(E, k, H, I, g, bg, bd)
    bank = quantize_bank_gpu(E, d, seed, device)  # one layer's worth of distinct experts, pinned
    specs = [LayerSpec(d, bank, synth.bank_permutation(seed, l, E).tolist()) for l in range(n_layers)]
    st = Streamer(specs, S, max_tokens=T, device=device)
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


def ffn_graph_time(st, cfg, snaps, reps, device):
    """Time the FFN alone: a CUDA graph of the 48 layers' moe_expert_ffn calls
    (each with its layer's routing from one decode step), replayed `reps`
    times; returns microseconds per layer."""
    import torch

    from streamed_quantized_expert_b200 import ops

    n_layers, E, k, H, I, g, bg, bd, T, S, _ = cfg
    y = torch.zeros((T, H), dtype=torch.float32, device=device)
    g_ = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)
    with torch.cuda.graph(g_, stream=cap):
        cs = torch.cuda.current_stream(device)
        for l in range(n_layers):
            sn = snaps[l]
            ops.moe_expert_ffn(sn["x"], T, st.layers[l].desc, st.pool_of(l), st.n_slots_of(l), st.table_dev[l],
                               sn["ids"], sn["w"], sn["offsets"], sn["pairs"], sn["meta"][2:], sn["meta"][0:1], None,
                               0, E, y, st.ws, st.ws_bytes, st.dev_err, cs)
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
    seed = 1000 * rank
    st = build_streamer(cfg, seed, device)
    steps_total = args.warmup + args.steps
    # the popularity bias of the logits and the initially resident experts come from the same seed
    x, logits = make_inputs(cfg, seed, steps_total + 1, device)
    s = st.stream

    def step(i, x_src, lg_src):
        for l in range(n_layers):
            st.decode_layer(l, x_src[i, l], lg_src[i, l], T)

    for i in range(args.warmup):
        step(i, x, logits)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()

    inst0, bytes0, l0 = st.installs, st.installed_bytes, st.launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize(device)
        e0.record(s)
        for i in range(args.warmup, steps_total):
            step(i, x, logits)
        e1.record(s)
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1)
        launches = st.launches - l0
        installs, inst_bytes = st.installs - inst0, st.installed_bytes - bytes0

        # one more (untimed) step whose per-layer routing is kept for the FFN-only replay
        snaps = []
        for l in range(n_layers):
            st.decode_layer(l, x[steps_total, l], logits[steps_total, l], T)
            snaps.append({"x": x[steps_total, l], "ids": st.ids.clone(), "w": st.w.clone(),
                          "offsets": st.offsets.clone(), "pairs": st.pairs.clone(), "meta": st.meta.clone()})
        torch.cuda.synchronize(device)
        n_unique = sum(int(sn["meta"][0].item()) for sn in snaps) / n_layers
        ffn_us = ffn_graph_time(st, cfg, snaps, args.ffn_reps, device)
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    err = st.check_dev_err()

    # e2e: inputs from pinned host memory copied in, y of every layer read back, same K steps
    xh, lgh = make_inputs(cfg, seed, args.steps, device, pinned=True, step0=steps_total + 1)
    yh = torch.empty((args.steps, n_layers, T, H), dtype=torch.float32).pin_memory()
    xd = torch.empty((n_layers, T, H), dtype=torch.int16, device=device)
    lgd = torch.empty((n_layers, T, E), dtype=torch.float32, device=device)
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
            y = st.decode_layer(l, xd[l], lgd[l], T)
            with torch.cuda.stream(s):
                yh[i, l].copy_(y, non_blocking=True)
    f1.record(s)
    torch.cuda.synchronize(device)
    e2e_ms = f0.elapsed_time(f1)
    t = torch.tensor([e2e_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_ms_max = float(t.item())

    if rank != 0:
        return None
    hbm_peak, tf_peak, peak_kind = peaks()
    tokens = args.steps * T * world
    from streamed_quantized_expert_b200 import ops as _ops

    slot_b = _ops.moe_slot_bytes(_ops.desc(E, k, H, I, g, bg, bd))
    ffn_bytes = n_unique * slot_b + T * H * 2 + T * H * 4
    achieved = ffn_bytes / (ffn_us * 1e-6) / 1e9
    flops_per_ffn = 2.0 * T * k * 3 * H * I
    out = {
        "metric": METRIC,
        "value": round(tokens / (ms_max / 1e3), 3),
        "unit": "tok/s (whole path: route+sort+lookup+installs+FFN+combine, %d layers)" % n_layers,
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
                   "parallelism": f"replicas x{world} (independent token streams)"},
        "ffn": {"tok_s_equiv": round(T / (n_layers * ffn_us * 1e-6), 1),
                "us_per_layer": round(ffn_us, 3),
                "hbm_gbs": round(achieved, 1),
                "tflops": round(flops_per_ffn / (ffn_us * 1e-6) / 1e12, 3),
                "how": "CUDA graph of the %d layers' moe_expert_ffn calls, replayed %d times, CUDA events" %
                       (n_layers, args.ffn_reps)},
        "installs": {"experts": installs, "per_token": round(installs / max(args.steps * T, 1), 2),
                     "miss_rate": round(installs / max(args.steps * n_layers * T * k, 1), 4),
                     "bytes": inst_bytes},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": None,
                     "kernel": "moe_expert_ffn (gate/up+SwiGLU kernel + down+combine kernel), per layer",
                     "bytes_per_launch": int(ffn_bytes), "peak_kind": peak_kind},
        "gpu_launches": launches,
        "dev_err": err,
        "clocks": clk.summary(),
        "e2e": {"value": round(tokens / (e2e_ms_max / 1e3), 3), "unit": "tok/s",
                "h2d_bytes_per_step": n_layers * (T * H * 2 + T * E * 4),
                "d2h_bytes_per_step": n_layers * T * H * 4},
    }
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg, seed, samples=args.cpu_layers)
    return out


# ---------------------------------------------------------------------------
# oracle (CPU) timing
# ---------------------------------------------------------------------------
def cpu_baseline(cfg, seed, samples=2, as_reference=False):
    """The oracle as it stands, single-threaded, on a bounded sample: `samples`
    layers of one decode step (route, sort, lookup, FFN+combine; the experts'
    slot bytes are prepared beforehand by the oracle's quantizer)."""
    import numpy as np

    import oracle as orc
    from streamed_quantized_expert_b200 import synth

    n_layers, E, k, H, I, g, bg, bd, T, S, _ = cfg
    samples = max(1, min(samples, n_layers))
    prep = []
    for l in range(samples):
        x = synth.activations(seed, l, T, H)
        logits = synth.router_logits(seed, l, T, E)
        ids, _, _ = orc.route(logits, k)
        slots = [None] * E
        for e in np.unique(ids):
            slots[int(e)] = orc.build_slot(*synth.expert_weights(seed, int(e), H, I), g, bg, bd)
        table = np.full(E, -1, np.int32)
        table[np.unique(ids)] = np.arange(np.unique(ids).size)
        prep.append((x, logits, slots, table))
    t0 = time.perf_counter()
    for x, logits, slots, table in prep:
        ids, w, _ = orc.route(logits, k)
        off, pairs, active = orc.sort(ids, E)
        orc.slot_lookup(table, active, 0, E, S)
        orc.expert_ffn(x, H, I, g, bg, bd, ids, w, slots)
    dt = time.perf_counter() - t0
    per_token_s = dt / samples * n_layers / T
    return {"value": round(1.0 / per_token_s, 6), "unit": "tok/s", "cores": 1, "kind": "oracle",
            "sample": f"{samples} of {n_layers} layers of one {T}-token decode step (route+sort+lookup+FFN), "
                      f"scaled to {n_layers} layers; {dt:.2f} s of CPU time"}


def run_reference(args, rank):
    if rank != 0:
        return None
    cfg = CONFIGS[args.config]
    n_layers, E, k, H, I, g, bg, bd, T, S, desc_txt = cfg
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(cfg, 7 + i, samples=1)
        if i >= args.warmup:
            vals.append(r)
    v = statistics.mean(r["value"] for r in vals)
    return {"metric": METRIC, "impl": "reference", "value": v, "unit": "tok/s (whole path, 48 layers)",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * T / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic", "config": {"workload": desc_txt},
            "cpu_baseline": {"value": v, "unit": "tok/s", "cores": 1, "kind": "oracle",
                             "sample": "per step: 1 of 48 layers of one decode token, scaled to 48 layers"},
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="decode")
    ap.add_argument("--cpu-layers", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ffn-reps", type=int, default=20)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (small profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.layers:
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
        out = run_ours(args, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
