"""Benchmark of the sparse-MoE FFN step on B200.

Default workload (decode): the full-size layer (d=2048, f=768, 512 routed
experts, top-10 plus 1 shared, 2-bit block-32 fp16-scale weights, Zipf(1.1)
routing) at T=1, run for 48 layers in a row, every layer with its own seeded
input tokens, router, shared expert and 512 experts in a 24,576-slot pool
(36.2 GB) behind a slot table whose 4,500 most popular experts sit in slots
0..4,499. (Chaining x_{l+1} = x_l + y_l through random-weight layers with no
normalisation diverges within three layers, after which the router no longer
follows the seeded routing; each layer therefore reads its own seeded x_l.)
One step = one pass of all 48 layers; the 48 layers' weights (~1 GB touched
per step) do not fit in the 126 MB L2, so every layer reads its weights from
HBM.

--workload prefill: one full-size layer at T=8192 (81,920 token-expert pairs,
Zipf-skewed over 512 experts), the prefill chunk of the pages.

Prints one JSON line (rank 0). --impl reference times the fp64 CPU oracle on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE decode tok/s & expert-weight GB/s vs HBM peak (2-bit, top-10 of 512)"
LAYERS = 48
HOT = 4500
SEED = 0
KERNELS_PER_LAYER_DECODE = 1  # one fused decode-layer kernel
# dram__bytes_read.sum + dram__bytes_write.sum of one fused decode-layer launch
# (T=1, 2-bit) from an ncu capture of the current kernel, or None when the
# kernel has changed since the last capture (the last one, of the revision
# before the routing step moved ahead of the shared expert's stages, read
# 20,537,600 B and wrote 256 B per launch)
DECODE_LAYER_DRAM_BYTES = None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.device = device
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "out", "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce_max(v: float, world: int) -> float:
    """Largest value over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ workload

class DecodeStack:
    """48 layers of the full-size decode layer, T tokens, pools on the device."""

    def __init__(self, T=1, bits=2, layers=LAYERS, seed=SEED):
        import torch
        from bit_expert_ffn_router_b200 import moe as M
        from bit_expert_ffn_router_b200 import synth
        self.M, self.torch = M, torch
        self.T, self.L = T, layers
        self.cfg = M.FULL.replace(bits=bits, out_fp32=0)
        cfg = self.cfg
        self.lay = M.expert_layout(cfg)
        self.stride = self.lay["bytes"]
        self.n_slots = layers * cfg.E
        dev = "cuda"
        # pool: uniform random code bytes, then fp16 U(0.005, 0.02) scales in the scale sections
        self.pool = torch.empty(self.n_slots, self.stride, dtype=torch.uint8, device=dev)
        synth.fill_random_bytes_(self.pool, seed + 11)
        self.shared = torch.empty(layers, self.stride, dtype=torch.uint8, device=dev)
        synth.fill_random_bytes_(self.shared, seed + 12)
        for name, seedoff in (("gu_scales", 13), ("dn_scales", 14)):
            lo = self.lay[name]
            n = (2 * cfg.f * (cfg.d // 32) if name == "gu_scales" else cfg.d * (cfg.f // 32)) * 2
            for s0 in range(0, self.n_slots, 2048):
                s1 = min(s0 + 2048, self.n_slots)
                synth.fill_scales_(self.pool[s0:s1, lo:lo + n], seed + seedoff * 100003 + s0)
            synth.fill_scales_(self.shared[:, lo:lo + n], seed + seedoff)
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 15)
        self.wr = torch.randn(layers, cfg.E, cfg.d, generator=g, device=dev) * 0.02
        hot = HOT * layers // LAYERS  # the hot share of the pool stays 4,500 / 24,576
        self.slot_of = torch.from_numpy(synth.hot_slot_table(layers, cfg.E, hot, seed)).to(dev)
        bias = np.stack([synth.bias_from_sets(synth.zipf_sets(T, cfg.E, cfg.k, seed + 1000 * l), cfg.E)
                         for l in range(layers)])
        self.bias = torch.from_numpy(bias).to(dev)
        self.x_host = np.stack([synth.activations(T, cfg.d, seed + 1000 * l + 16) for l in range(layers)])
        self.x_in = torch.from_numpy(self.x_host.view(np.int16)).to(dev).view(torch.bfloat16)  # [L, T, d]
        self.y_out = torch.empty(layers, T, cfg.d, dtype=torch.bfloat16, device=dev)
        self.ws = M.workspace(cfg, T)
        self.ctx = M.Context(torch.cuda.current_device())
        self.graph = None
        # unique experts per layer (for the byte count)
        idx = [np.argsort(-bias[l], axis=1)[:, :cfg.k] for l in range(layers)]
        self.uniq = [len(np.unique(i)) for i in idx]
        self.expert_bytes_step = sum((u + cfg.n_shared) * self.stride for u in self.uniq)
        self.router_bytes_step = layers * cfg.E * cfg.d * 4

    def layer(self, l, x, y):
        cfg = self.cfg
        self.ctx.layer_forward(cfg, x, self.T, self.wr[l], self.bias[l], self.slot_of[l * cfg.E:(l + 1) * cfg.E],
                               self.n_slots, self.pool, self.stride, self.shared[l], self.ws, y)

    def step_eager(self):
        for l in range(self.L):
            self.layer(l, self.x_in[l], self.y_out[l])
        return self.y_out

    def prepare(self):
        """One prepared moe_layer_forward per layer (arguments marshalled once), as
        a host program driving the C ABI would hold them."""
        cfg = self.cfg
        self.prepared = [
            (self.ctx.prepare_layer_forward(cfg, self.T, self.wr[l], self.bias[l],
                                            self.slot_of[l * cfg.E:(l + 1) * cfg.E], self.n_slots, self.pool,
                                            self.stride, self.shared[l], self.ws),
             self.x_in[l], self.y_out[l])
            for l in range(self.L)]

    def step_prepared(self):
        for call, x, y in self.prepared:
            call(x, y)
        return self.y_out

    def capture(self):
        torch = self.torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step_eager()  # warm (attributes, lazy init) outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.out = self.step_eager()
        torch.cuda.synchronize()

    def time_expert_ffn(self, reps=3):
        """CUDA-event time of the decode expert kernels (gate/up + down/combine) per layer."""
        torch, M, cfg = self.torch, self.M, self.cfg
        st = torch.cuda.current_stream()
        logits = torch.empty(self.T, cfg.E, device="cuda")
        idx = torch.empty(self.T, cfg.k, dtype=torch.int32, device="cuda")
        gate = torch.empty(self.T, cfg.k, device="cuda")
        groups = []
        wss = []
        for l in range(self.L):
            ws = M.workspace(cfg, self.T)
            self.ctx.router_topk(cfg, self.x_in[l], self.wr[l], self.bias[l], self.T, logits, idx, gate)
            groups.append(self.ctx.group_tokens(cfg, idx, gate, self.T, self.slot_of[l * cfg.E:(l + 1) * cfg.E],
                                                self.n_slots, ws))
            wss.append(ws)
        y = torch.empty(self.T, cfg.d, dtype=torch.bfloat16, device="cuda")
        evs = []
        for r in range(reps + 1):
            for l in range(self.L):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(st)
                self.ctx.expert_ffn(cfg, self.x_in[l], groups[l], self.pool, self.stride, self.shared[l], wss[l], None,
                                    y)
                b.record(st)
                if r > 0:
                    evs.append((a, b, l))
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b, _ in evs]
        bytes_ = [(self.uniq[l] + cfg.n_shared) * self.stride for _, _, l in evs]
        return float(np.mean(ms)), float(np.mean(bytes_))


KERNELS_PER_LAYER_PREFILL = 9  # router GEMM, top-k, 3 grouping, x gather, 2 grouped GEMMs, combine


class PrefillLayer:
    """One full-size layer at T tokens (prefill chunk): 512 experts in a slot
    pool behind a shuffled slot table, Zipf routing, bf16 output."""

    def __init__(self, T=8192, bits=2, seed=SEED):
        import torch
        from bit_expert_ffn_router_b200 import moe as M
        from bit_expert_ffn_router_b200 import synth
        self.M, self.torch = M, torch
        self.T = T
        self.cfg = M.FULL.replace(bits=bits, out_fp32=0)
        cfg = self.cfg
        self.lay = M.expert_layout(cfg)
        self.stride = self.lay["bytes"]
        self.n_slots = cfg.E
        dev = "cuda"
        self.pool = torch.empty(self.n_slots, self.stride, dtype=torch.uint8, device=dev)
        synth.fill_random_bytes_(self.pool, seed + 21)
        self.shared = torch.empty(1, self.stride, dtype=torch.uint8, device=dev)
        synth.fill_random_bytes_(self.shared, seed + 22)
        for name, seedoff in (("gu_scales", 23), ("dn_scales", 24)):
            lo = self.lay[name]
            n = (2 * cfg.f * (cfg.d // 32) if name == "gu_scales" else cfg.d * (cfg.f // 32)) * 2
            synth.fill_scales_(self.pool[:, lo:lo + n], seed + seedoff)
            synth.fill_scales_(self.shared[:, lo:lo + n], seed + seedoff + 1)
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 25)
        self.wr = torch.randn(cfg.E, cfg.d, generator=g, device=dev) * 0.02
        self.slot_of = torch.from_numpy(synth.rng(seed + 26).permutation(cfg.E).astype(np.int32)).to(dev)
        self.sets = synth.zipf_sets(T, cfg.E, cfg.k, seed)
        self.bias = torch.from_numpy(synth.bias_from_sets(self.sets, cfg.E)).to(dev)
        self.x_host = synth.activations(T, cfg.d, seed + 27)
        self.x = torch.from_numpy(self.x_host.view(np.int16)).to(dev).view(torch.bfloat16)
        self.y = torch.empty(T, cfg.d, dtype=torch.bfloat16, device=dev)
        self.ws = M.workspace(cfg, T)
        self.ctx = M.Context(torch.cuda.current_device())
        counts = np.bincount(np.asarray(self.sets).reshape(-1), minlength=cfg.E)
        self.load = {"max": int(counts.max()), "median": float(np.median(counts)), "min": int(counts.min()),
                     "experts_lt16": int((counts < 16).sum()), "experts_ge128": int((counts >= 128).sum())}
        self.flops = 6 * cfg.d * cfg.f * (T * cfg.k + T * cfg.n_shared)
        self.graph = None

    def step(self):
        self.ctx.layer_forward(self.cfg, self.x, self.T, self.wr, self.bias, self.slot_of, self.n_slots, self.pool,
                               self.stride, self.shared[0], self.ws, self.y)
        return self.y

    def capture(self):
        torch = self.torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        torch.cuda.synchronize()

    def time_parts(self, reps=5):
        """CUDA-event time of each entry point of the unfused path (ms)."""
        torch, M, cfg, T = self.torch, self.M, self.cfg, self.T
        st = torch.cuda.current_stream()
        logits = torch.empty(T, cfg.E, device="cuda")
        idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
        gate = torch.empty(T, cfg.k, device="cuda")
        ws = M.workspace(cfg, T)
        z = torch.empty(T * cfg.k + T, cfg.d, device="cuda")
        parts = {"router_topk": [], "group": [], "expert_ffn": [], "combine": []}
        g = None
        for r in range(reps + 1):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            ev[0].record(st)
            self.ctx.router_topk(cfg, self.x, self.wr, self.bias, T, logits, idx, gate)
            ev[1].record(st)
            g = self.ctx.group_tokens(cfg, idx, gate, T, self.slot_of, self.n_slots, ws)
            ev[2].record(st)
            self.ctx.expert_ffn(cfg, self.x, g, self.pool, self.stride, self.shared[0], ws, z_rows=z)
            ev[3].record(st)
            self.ctx.combine(cfg, g, z, self.x, T, self.y)
            ev[4].record(st)
            torch.cuda.synchronize()
            if r > 0:
                for i, k in enumerate(parts):
                    parts[k].append(ev[i].elapsed_time(ev[i + 1]))
        return {k: float(np.median(v)) for k, v in parts.items()}


def run_prefill(args):
    import torch
    world, rank, local = dist_setup()
    hbm, tf, tf_s, peak_kind = peaks()
    pl = PrefillLayer(T=args.tokens if args.tokens > 8 else 8192, bits=args.bits)
    pl.capture()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        pl.graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            pl.graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_max = allreduce_max(e0.elapsed_time(e1), world)
    ms_step = ms_max / args.steps
    value = pl.T * args.steps * world / (ms_max / 1e3)

    parts = pl.time_parts()
    ffn_ms = parts["expert_ffn"]
    achieved = pl.flops / (ffn_ms / 1e3) / 1e12

    xh = torch.from_numpy(pl.x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    for _ in range(2):
        pl.x.copy_(xh, non_blocking=True)
        yh.copy_(pl.step(), non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, args.steps // 4)
    e2.record(stream)
    for _ in range(n_e2e):
        pl.x.copy_(xh, non_blocking=True)
        yh.copy_(pl.step(), non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(e2.elapsed_time(e3), world)
    e2e_value = pl.T * n_e2e * world / (e2e_ms / 1e3)

    res = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": f"tokens/s (one MoE layer, prefill chunk T={pl.T})",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"u{args.bits} codes -> f16 x f16 tcgen05, f32 accumulate",
        "data": "synthetic (seeded; random-init weights of the stated shapes)",
        "config": {
            "workload": f"prefill layer d=2048 f=768 E=512 top-10 + 1 shared, T={pl.T} "
                        f"({pl.T * pl.cfg.k} pairs), {args.bits}-bit block-32 fp16-scale, Zipf(1.1) routing",
            "global_batch": pl.T * world, "seq_len": pl.T, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (0.76-1.06 GB of expert weights per layer)",
            "expert_load": pl.load, "parts_ms": {k: round(v, 4) for k, v in parts.items()},
            "useful_gflop": round(pl.flops / 1e9, 1),
        },
        "roofline": {
            "kernel": "prefill expert FFN call (tile table + x gather + gate/up and down tcgen05 grouped GEMMs; "
                      "the GEMMs are ~95% of it), useful FLOPs",
            "bound": "tensor", "achieved": round(achieved, 1), "peak": tf, "unit": "TFLOP/s",
            "frac": round(achieved / tf, 4), "peak_source": f"{peak_kind} bf16 burst (fp16 has the same dense rate)",
            "traffic": None, "avg_launch_us": round(ffn_ms * 1e3, 2), "flops_per_launch": pl.flops,
        },
        "e2e": {"value": round(e2e_value, 1), "unit": f"tokens/s (one MoE layer, prefill chunk T={pl.T})",
                "h2d_bytes_per_step": pl.T * pl.cfg.d * 2, "d2h_bytes_per_step": pl.T * pl.cfg.d * 2,
                "how": "pinned host x -> moe_layer_forward -> pinned host y (bf16), CUDA events"},
        "gpu_launches": KERNELS_PER_LAYER_PREFILL * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_prefill(pl, args.cpu_tokens)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_ours(args):
    import torch
    world, rank, local = dist_setup()
    hbm, tf, tf_s, peak_kind = peaks()
    st = DecodeStack(T=args.tokens, bits=args.bits, layers=args.layers)
    st.capture()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        st.graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            st.graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = allreduce_max(ms, world)
    ms_step = ms_max / args.steps
    tokens = st.T * args.steps * world
    value = tokens / (ms_max / 1e3 * LAYERS / st.L)  # per 48-layer stack (st.L < 48 only when profiling)

    # The dominant (and only) kernel of the timed step is the fused decode-layer
    # kernel, one launch per layer: its average launch time over the timed
    # region and its algorithmic bytes per launch (the selected experts'
    # records, the router matrix, x and y).
    layer_launch_s = ms_step / 1e3 / st.L
    layer_bytes = (st.expert_bytes_step + st.router_bytes_step) / st.L + 2 * st.T * st.cfg.d * 2
    achieved = layer_bytes / layer_launch_s / 1e9
    # side measurement: the expert FFN alone (grouping given), cold weights
    ffn_ms, ffn_bytes = st.time_expert_ffn()

    # end to end through the public API: pinned host x in, 48 eager layer calls
    # (each layer's arguments marshalled once, before the timed region), host y out
    xh = torch.from_numpy(st.x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    how = "48 eager moe_layer_forward calls (arguments marshalled once per layer)"
    try:
        st.prepare()
        step = st.step_prepared
        st.x_in.copy_(xh, non_blocking=True)
        step()
        torch.cuda.synchronize()
    except st.M.MoeError:
        raise
    except Exception as exc:  # the binding's prepared form failed: time the plain calls instead
        print(f"prepared calls unavailable ({exc!r}); timing the plain binding calls", file=sys.stderr)
        step, how = st.step_eager, "48 eager moe_layer_forward calls"
    for _ in range(2):
        st.x_in.copy_(xh, non_blocking=True)
        out = step()
        yh.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    n_e2e = max(3, args.steps // 4)
    for _ in range(n_e2e):
        st.x_in.copy_(xh, non_blocking=True)
        out = step()
        yh.copy_(out, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(e2.elapsed_time(e3), world)
    e2e_value = st.T * n_e2e * world / (e2e_ms / 1e3 * LAYERS / st.L)

    layer_us = ms_step * 1e3 / st.L
    expert_gbs_layer = st.expert_bytes_step / (ms_step / 1e3) / 1e9
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s (48-layer MoE stack)",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u2 codes x bf16 act, f32 accumulate",
        "data": "synthetic (seeded; random-init weights of the stated shapes)",
        "config": {
            "workload": f"decode layer d=2048 f=768 E=512 top-10 + 1 shared, T={st.T}, "
                        f"{args.bits}-bit block-32 fp16-scale, Zipf(1.1) routing; {st.L} distinct layers per step",
            "global_batch": st.T * world, "seq_len": 1, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (48 layers, ~1 GB touched per step)",
            "layer_us": round(layer_us, 3),
            "layer_tok_s": round(1e6 / layer_us * st.T, 1),
            "expert_gbs_in_stack": round(expert_gbs_layer, 1),
            "expert_bytes_per_step": st.expert_bytes_step,
            "router_bytes_per_step": st.router_bytes_step,
            "uniq_experts_per_layer": round(float(np.mean(st.uniq)), 2),
        },
        "roofline": {
            "kernel": "fused decode layer kernel (router, top-k, grouping, experts, combine), one launch per layer",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": f"{peak_kind} copy bandwidth",
            "traffic": DECODE_LAYER_DRAM_BYTES if st.T == 1 and args.bits == 2 else None,
            "avg_launch_us": round(layer_launch_s * 1e6, 3), "bytes_per_launch": round(layer_bytes),
            "expert_ffn_only": {"avg_launch_us": round(ffn_ms * 1e3, 3), "expert_bytes": ffn_bytes,
                                "gbs": round(ffn_bytes / (ffn_ms / 1e3) / 1e9, 1)},
        },
        "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s (48-layer MoE stack)",
                "h2d_bytes_per_step": st.L * st.T * st.cfg.d * 2, "d2h_bytes_per_step": st.L * st.T * st.cfg.d * 2,
                "how": f"pinned host x (48 layers' tokens) -> {how} -> pinned host y, CUDA events"},
        "gpu_launches": KERNELS_PER_LAYER_DECODE * st.L * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(st, min(args.cpu_layers, st.L))
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_layer_inputs(st, l):
    """Host copies of layer l's inputs (router, bias, the records it selects)."""
    from oracle import moe_oracle as O
    cfg = st.cfg
    wr = st.wr[l].cpu().numpy()
    bias = st.bias[l].cpu().numpy()
    sel = np.unique(np.argsort(-bias, axis=1)[:, :cfg.k])
    slot_of = st.slot_of[l * cfg.E:(l + 1) * cfg.E].cpu().numpy()
    recs = {int(e): st.pool[int(slot_of[e])].cpu().numpy() for e in sel}
    shared = st.shared[l].cpu().numpy()
    return wr, bias, recs, shared


def cpu_baseline(st, n_layers):
    """The fp64 oracle, as it stands, on a sample of the stack's layers (T tokens each)."""
    from oracle import moe_oracle as O
    import threadpoolctl
    cfg = st.cfg
    inputs = [oracle_layer_inputs(st, l) for l in range(n_layers)]
    t0 = time.perf_counter()
    for l, (wr, bias, recs, shared) in enumerate(inputs):
        cache = O.ExpertCache(lambda e, r=recs: O.sections_from_record(r[e], cfg.d, cfg.f, cfg.bits),
                              cfg.d, cfg.f, cfg.bits)
        sh = O.expert_weights(O.sections_from_record(shared, cfg.d, cfg.f, cfg.bits), cfg.d, cfg.f, cfg.bits)
        O.layer_forward(st.x_host[l], wr, cfg.k, cache, sh, bias=bias)
    dt = time.perf_counter() - t0
    per_layer = dt / n_layers
    info = threadpoolctl.threadpool_info()
    cores = max([i.get("num_threads", 1) for i in info] + [1])
    return {"value": round(st.T / (per_layer * LAYERS), 4), "unit": "tokens/s (48-layer MoE stack)",
            "cores": cores, "kind": "oracle",
            "sample": f"{n_layers} of 48 layers at T={st.T} (fp64 numpy oracle, {dt:.1f} s), scaled to 48 layers"}


def prefill_oracle_inputs(pl, tokens):
    cfg = pl.cfg
    sel = np.unique(np.asarray(pl.sets)[tokens].reshape(-1))
    slot_of = pl.slot_of.cpu().numpy()
    recs = {int(e): pl.pool[int(slot_of[e])].cpu().numpy() for e in sel}
    return (pl.x_host[tokens], pl.wr.cpu().numpy(), pl.bias.cpu().numpy()[tokens], recs,
            pl.shared[0].cpu().numpy())


def cpu_baseline_prefill(pl, n_tokens):
    """The fp64 oracle, as it stands, on the first n_tokens of the chunk."""
    from oracle import moe_oracle as O
    import threadpoolctl
    cfg = pl.cfg
    x, wr, bias, recs, shared = prefill_oracle_inputs(pl, np.arange(n_tokens))
    t0 = time.perf_counter()
    cache = O.ExpertCache(lambda e: O.sections_from_record(recs[e], cfg.d, cfg.f, cfg.bits), cfg.d, cfg.f, cfg.bits)
    sh = O.expert_weights(O.sections_from_record(shared, cfg.d, cfg.f, cfg.bits), cfg.d, cfg.f, cfg.bits)
    O.layer_forward(x, wr, cfg.k, cache, sh, bias=bias)
    dt = time.perf_counter() - t0
    cores = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])
    return {"value": round(n_tokens / dt, 3), "unit": f"tokens/s (one MoE layer, prefill chunk T={pl.T})",
            "cores": cores, "kind": "oracle",
            "sample": f"first {n_tokens} of {pl.T} tokens of the chunk (fp64 numpy oracle, {dt:.1f} s)"}


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, a bounded sample per step."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.workload == "prefill":
        return run_reference_prefill(args, world)
    from oracle import moe_oracle as O
    from bit_expert_ffn_router_b200 import synth
    import threadpoolctl
    cfg_d, cfg_f, E, k, bits = 2048, 768, 512, 10, args.bits
    T = args.tokens
    layers_per_step = 2
    layers = []
    for l in range(layers_per_step):
        wr = synth.router_weights(E, cfg_d, SEED + 1000 * l + 1)
        bias = synth.bias_from_sets(synth.zipf_sets(T, E, k, SEED + 1000 * l), E)
        sel = np.unique(np.argsort(-bias, axis=1)[:, :k])
        secs = {int(e): synth.expert_sections(cfg_d, cfg_f, bits, SEED + 100 + 1000 * l + int(e)) for e in sel}
        shared = synth.expert_sections(cfg_d, cfg_f, bits, SEED + 99 + 1000 * l)
        x = synth.activations(T, cfg_d, SEED + 1000 * l + 16)
        layers.append((x, wr, bias, secs, shared))
    times = []
    for step in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for x, wr, bias, secs, shared in layers:
            cache = O.ExpertCache(lambda e, s=secs: s[e], cfg_d, cfg_f, bits)
            sh = O.expert_weights(shared, cfg_d, cfg_f, bits)
            O.layer_forward(x, wr, k, cache, sh, bias=bias)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt / layers_per_step)
    per_layer = float(np.mean(times))
    value = T / (per_layer * LAYERS)
    cores = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])
    sample = f"{layers_per_step} of 48 layers per step at T={T}, scaled to 48 layers"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s (48-layer MoE stack)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_layer * LAYERS * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"decode layer d=2048 f=768 E=512 top-10 + 1 shared, T={T}, {bits}-bit; "
                               f"48 distinct layers per step (oracle sample)", "global_batch": T, "seq_len": 1,
                   "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s (48-layer MoE stack)", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "tokens/s (48-layer MoE stack)", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference_prefill(args, world):
    """Reference arm of the prefill workload: the oracle on a bounded token sample per step."""
    from oracle import moe_oracle as O
    from bit_expert_ffn_router_b200 import synth
    import threadpoolctl
    d, f, E, k, bits, T = 2048, 768, 512, 10, args.bits, 8192
    n = 4  # tokens per step: keeps --steps 50 --warmup 5 within a few minutes
    sets = synth.zipf_sets(T, E, k, SEED)[:n]
    bias = synth.bias_from_sets(sets, E)
    wr = synth.router_weights(E, d, SEED + 1)
    x = synth.activations(T, d, SEED + 27)[:n]
    sel = np.unique(np.asarray(sets).reshape(-1))
    secs = {int(e): synth.expert_sections(d, f, bits, SEED + 100 + int(e)) for e in sel}
    shared = synth.expert_sections(d, f, bits, SEED + 99)
    times = []
    for step in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cache = O.ExpertCache(lambda e: secs[e], d, f, bits)
        O.layer_forward(x, wr, k, cache, O.expert_weights(shared, d, f, bits), bias=bias)
        if step >= args.warmup:
            times.append(time.perf_counter() - t0)
    value = n / float(np.mean(times))
    cores = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])
    unit = f"tokens/s (one MoE layer, prefill chunk T={T})"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(float(np.mean(times)) * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"prefill layer d=2048 f=768 E=512 top-10 + 1 shared, T={T}, {bits}-bit "
                               f"(oracle on {n} tokens per step)", "global_batch": n, "seq_len": T,
                   "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 3), "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"{n} of {T} tokens per step"},
        "e2e": {"value": round(value, 3), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--tokens", type=int, default=1)
    ap.add_argument("--bits", type=int, default=2)
    ap.add_argument("--cpu-layers", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="decode", choices=["decode", "prefill"])
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="decode: layers in the stack (fewer only to profile a small case)")
    ap.add_argument("--cpu-tokens", type=int, default=32, help="prefill: oracle sample size")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefill":
        run_prefill(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
