"""Benchmark of the sparse-MoE FFN step on B200.

Default workload (decode): the full-size layer (d=2048, f=768, 512 routed
experts, top-10 plus 1 shared, 2-bit block-32 fp16-scale weights, Zipf(1.1)
routing) at T=1, run for 48 layers in a row by moe_stack_forward (one launch
per step): layer l + 1 reads layer l's output (a residual stream
y_l = x_l + moe(x_l)), every layer has its own router, shared expert, Zipf
popularity and 512 experts in a 24,576-slot pool (36.2 GB) behind a slot
table whose 4,500 most popular experts sit in slots 0..4,499. The seeded
bias (+20 on each token's Zipf-drawn experts, against router logits of
about +-2) keeps the routing on the seeded draw along the chain. One step =
one pass of all 48 layers; the 48 layers' weights (~1 GB touched per step)
do not fit in the 126 MB L2, so every layer reads its weights from HBM.

The default line also carries, under config.extras, the other
configurations: the same layers as 48 single-layer launches, the 48-layer
stack at the verify width T=4 over 256 consecutive steps with 70 % of each
token position's experts kept from the step before, the 3-bit stack at
T = 1..4 (64 correlated steps each) and the T=8192 prefill chunk (2- and
3-bit).

--workload stack: that T=4 (--tokens 4) correlated stack as the headline.
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
# dram__bytes_read.sum + dram__bytes_write.sum of one decode stack launch from
# an ncu capture of the current kernel, keyed by (T, bits, layers, correlated
# workload), scaled to the stack's layers when the capture ran fewer; absent
# until a capture of the current kernel exists
DECODE_STACK_DRAM_BYTES = {
    # 8-layer capture: 163.58 MB read + 3.64 MB written, x 48 / 8
    (1, 2, 48, False): 1003.3e6,
}
STACK_X_SCALE = 2.0 ** -5


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

def cpu_info():
    """Host cores and CPU model (the oracle baseline runs there)."""
    model = ""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "model": model}


def make_pool(bits, layers=LAYERS, seed=SEED):
    """The stack's device tensors: a layers*512-slot pool of full-size records
    (uniform random codes, fp16 U(0.005, 0.02) scales), one shared expert per
    layer, the routers W_r [L, 512, 2048] ~ N(0, 0.02^2) and the hot-slot table
    (the 4,500 most popular experts of the 48 layers in slots 0..4,499)."""
    import torch
    from bit_expert_ffn_router_b200 import moe as M
    from bit_expert_ffn_router_b200 import synth
    cfg = M.FULL.replace(bits=bits, out_fp32=0, residual=1)
    lay = M.expert_layout(cfg)
    stride = lay["bytes"]
    n_slots = layers * cfg.E
    dev = "cuda"
    pool = torch.empty(n_slots, stride, dtype=torch.uint8, device=dev)
    synth.fill_random_bytes_(pool, seed + 11)
    shared = torch.empty(layers, stride, dtype=torch.uint8, device=dev)
    synth.fill_random_bytes_(shared, seed + 12)
    for name, seedoff in (("gu_scales", 13), ("dn_scales", 14)):
        lo = lay[name]
        n = (2 * cfg.f * (cfg.d // 32) if name == "gu_scales" else cfg.d * (cfg.f // 32)) * 2
        for s0 in range(0, n_slots, 2048):
            s1 = min(s0 + 2048, n_slots)
            synth.fill_scales_(pool[s0:s1, lo:lo + n], seed + seedoff * 100003 + s0)
        synth.fill_scales_(shared[:, lo:lo + n], seed + seedoff)
    g = torch.Generator(device=dev)
    g.manual_seed(seed + 15)
    wr = torch.randn(layers, cfg.E, cfg.d, generator=g, device=dev) * 0.02
    hot = HOT * layers // LAYERS  # the hot share of the pool stays 4,500 / 24,576
    slot_of = torch.from_numpy(synth.hot_slot_table(layers, cfg.E, hot, seed)).to(dev)
    return {"cfg": cfg, "bits": bits, "layers": layers, "lay": lay, "stride": stride, "n_slots": n_slots,
            "pool": pool, "shared": shared, "wr": wr, "slot_of": slot_of, "hot": hot}


class DecodeStack:
    """L chained full-size decode layers run by moe_stack_forward (one launch
    per step; layer l + 1 reads layer l's output, a residual stream y_l =
    x_l + moe(x_l)). Routing per layer follows a Zipf(1.1) popularity: one
    fixed draw (steps=1), or `steps` consecutive decode steps in which every
    token position keeps `keep` of its previous step's experts."""

    def __init__(self, pool, T=1, steps=1, keep=None, seed=SEED):
        import torch
        from bit_expert_ffn_router_b200 import moe as M
        from bit_expert_ffn_router_b200 import synth
        self.M, self.torch, self.p = M, torch, pool
        self.cfg = cfg = pool["cfg"]
        self.T, self.L = T, pool["layers"]
        L, E, k = self.L, cfg.E, cfg.k
        if keep is None:
            sets = np.stack([synth.zipf_sets(T, E, k, seed + 1000 * l) for l in range(L)])[None]  # [1, L, T, k]
        else:
            sets = np.stack([synth.correlated_sets(steps, T, E, k, keep, seed + 1000 * l) for l in range(L)],
                            axis=1)  # [S, L, T, k]
        self.sets = sets
        self.S = sets.shape[0]
        bias = np.zeros((self.S, L, T, E), dtype=np.float32)
        np.put_along_axis(bias, sets.astype(np.int64), np.float32(synth.BIAS), axis=3)
        self.bias = torch.from_numpy(bias).to("cuda")
        self.uniq = np.array([[len(np.unique(sets[s, l])) for l in range(L)] for s in range(self.S)])
        # x ~ N(0, 2^-10): with random-init experts a layer's update is then
        # about 1 % of the residual stream, which stays finite over 48 layers
        # (at N(0, 1) the SwiGLU terms overflow bf16 within five layers)
        self.x_host = synth.activations(T, cfg.d, seed + 16, scale=STACK_X_SCALE)
        self.x0 = torch.from_numpy(self.x_host.view(np.int16)).to("cuda").view(torch.bfloat16)
        self.y = torch.empty(L, T, cfg.d, dtype=torch.bfloat16, device="cuda")
        self.ws = M.stack_workspace(cfg, L, T)
        self.ctx = M.Context(torch.cuda.current_device())
        self.call = self.ctx.prepare_stack_forward(cfg, L, T, pool["wr"], pool["slot_of"], pool["n_slots"],
                                                   pool["pool"], pool["stride"], pool["shared"], self.ws)

    def step(self, s=0):
        self.call(self.x0, self.bias[s % self.S], self.y)
        return self.y

    def expert_bytes(self, s):
        return int((self.uniq[s % self.S] + self.cfg.n_shared).sum()) * self.p["stride"]

    def step_bytes(self, s):
        """Algorithmic bytes of one step: the records of the selected and
        shared experts, the routers and every layer's x and y."""
        cfg = self.cfg
        return self.expert_bytes(s) + self.L * cfg.E * cfg.d * 4 + self.L * 2 * self.T * cfg.d * 2


def time_steps(st, steps, warmup, world, local, first=0):
    """Device time (ms, max over ranks) of `steps` consecutive stack steps after
    `warmup` untimed ones, with the clocks sampled during the timed region."""
    import torch
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        st.step(first + i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            st.step(first + warmup + i)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    st.ctx.check_device_status() == 0 or sys.exit("device error in the timed steps")
    return allreduce_max(e0.elapsed_time(e1), world), clk.summary()


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


def workload_name(T, bits, layers=LAYERS, correlated=False):
    what = (f"48-layer stack at the verify width T={T}, 256 consecutive decode steps with routing temporally "
            f"correlated (each token position keeps 7 of its 10 experts from the step before)"
            if correlated else f"decode layer, T={T}")
    return (f"{what}: d=2048 f=768 E=512 top-10 + 1 shared, {bits}-bit block-32 fp16-scale, Zipf(1.1) routing, "
            f"{layers} chained layers per step (layer l+1 reads layer l's output), {layers * 512}-slot pool with "
            f"{HOT * layers // LAYERS} hot slots")


def stack_record(st, ms_total, steps, first, hbm, world):
    """Compact numbers of a timed run of stack steps [first, first + steps)."""
    idx = [(first + i) % st.S for i in range(steps)]
    ms_step = ms_total / steps
    ebytes = float(np.mean([st.expert_bytes(s) for s in idx]))
    sbytes = float(np.mean([st.step_bytes(s) for s in idx]))
    u = st.uniq[idx]
    return {
        "tok_s": round(st.T * steps * world / (ms_total / 1e3), 1),
        "ms_per_step": round(ms_step, 4), "layer_us": round(ms_step * 1e3 / st.L, 3),
        "uniq_experts_per_layer": {"mean": round(float(u.mean()), 2), "min": int(u.min()), "max": int(u.max())},
        "expert_gbs": round(ebytes / (ms_step / 1e3) / 1e9, 1),
        "expert_frac_of_hbm": round(ebytes / (ms_step / 1e3) / 1e9 / hbm, 4),
        "step_gbs": round(sbytes / (ms_step / 1e3) / 1e9, 1),
        "step_frac_of_hbm": round(sbytes / (ms_step / 1e3) / 1e9 / hbm, 4),
    }


def skip_record(st, pool, skip_from, steps=20):
    """The stack with low-ranked non-resident pairs left out (rank >= skip_from,
    slot >= the pool's hot slots): time per layer, the share of pairs left out,
    and the drift of the layer outputs from the plain stack's (relative L2 per
    token of y[l] = x_l + moe(x_l); layer 0 shows one step's effect, the last
    layer the effect compounded over the stack)."""
    import torch
    M, L, T = st.M, st.L, st.T
    cfg = st.cfg.replace(skip_from=skip_from, hot_slots=pool["hot"])
    call = st.ctx.prepare_stack_forward(cfg, L, T, pool["wr"], pool["slot_of"], pool["n_slots"], pool["pool"],
                                        pool["stride"], pool["shared"], st.ws)
    plain = st.step(0).clone().float()
    y = torch.empty_like(st.y)
    for _ in range(3):
        call(st.x0, st.bias[0], y)
    torch.cuda.synchronize()
    left = [float((st.ctx.layer_routing(cfg, T, st.ws, stack_layers=L, layer=l)["pair_pos"] < 0).float().mean())
            for l in range(L)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        call(st.x0, st.bias[0], y)
    e1.record()
    torch.cuda.synchronize()
    assert st.ctx.check_device_status() == M.OK
    ms = e0.elapsed_time(e1) / steps
    x0 = st.x0.float()
    d_moe0 = ((y[0].float() - plain[0]).norm(dim=-1) / (plain[0] - x0).norm(dim=-1)).max().item()
    d = ((y.float() - plain).norm(dim=-1) / plain.norm(dim=-1)).cpu().numpy()  # [L, T]
    return {"skip_from": skip_from, "hot_slots": int(pool["hot"]), "layer_us": round(ms * 1e3 / L, 3),
            "pairs_left_out": round(float(np.mean(left)), 4),
            "rel_drift_moe_layer0": float(f"{d_moe0:.3g}"),
            "rel_drift_y_last_layer": float(f"{d[-1].max():.3g}"), "rel_drift_y_max": float(f"{d.max():.3g}"),
            "how": "layer 0: the MoE term moe(x) = y - x against the plain stack's on the same input; "
                   "y: the layer outputs x_l + moe(x_l) after l skipping layers"}


def residency_record(st, pool, every=8, prior=8):
    """The hot set under a T=4 decode stream: moe_usage_count after every
    step; counts start at `prior` on the table's hot entries (the seeded
    hot set), lose an eighth (rounded down) at each adaptation, and every
    `every` steps the
    plan_swaps exchanges are carried out by moe_slot_swap. Reports the share
    of routed pairs whose expert sits in the pool's first `hot` slots with the
    table the stream started from (static) and with the adapted one, and the
    exchange cost."""
    import torch
    from bit_expert_ffn_router_b200 import residency as R
    M, cfg, ctx = st.M, st.cfg, st.ctx
    L, E, T, n_hot = st.L, cfg.E, st.T, pool["hot"]
    table = pool["slot_of"].view(-1)
    static = table.cpu().numpy().copy()
    cur = static.copy()
    counts = torch.from_numpy(np.where(static < n_hot, prior, 0).astype(np.int32)).cuda()
    hit_s = hit_a = 0.0
    n_sw, sw_ms = 0, 0.0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for s in range(st.S):
        st.step(s)
        ctx.usage_count(cfg, L, T, st.ws, counts)
        ex = [st.sets[s, l].reshape(-1) for l in range(L)]
        hit_s += R.hot_hit_rate(ex, static, E, n_hot)
        hit_a += R.hot_hit_rate(ex, cur, E, n_hot)
        if s % every == every - 1:
            a, b = R.plan_swaps(counts.cpu().numpy(), cur, n_hot)
            e0.record()
            ctx.slot_swap(cfg, pool["pool"], pool["stride"], table, pool["n_slots"], a, b)
            e1.record()
            torch.cuda.synchronize()
            sw_ms += e0.elapsed_time(e1)
            n_sw += a.size
            cur = R.apply_swaps(cur, a, b)
            counts.sub_(counts // 8)
    assert ctx.check_device_status() == M.OK
    assert np.array_equal(table.cpu().numpy(), cur)
    rec = pool["lay"]["bytes"]
    return {"hot_slots": int(n_hot), "steps": int(st.S), "adapt_every": every,
            "hot_hit_rate_static": round(hit_s / st.S, 4), "hot_hit_rate_adaptive": round(hit_a / st.S, 4),
            "swaps": int(n_sw), "swap_us_each": round(sw_ms * 1e3 / max(n_sw, 1), 2),
            "swap_gbs": round(4 * rec * n_sw / max(sw_ms, 1e-9) / 1e6, 1)}


def layer_call_record(st, steps, world):
    """The same stack as L separate moe_layer_forward launches (one CUDA graph
    per step): the single-layer entry point's speed."""
    import torch
    M, cfg, p = st.M, st.cfg, st.p
    ws = M.workspace(cfg, st.T)
    bias = st.bias[0]
    s = torch.cuda.Stream()  # the calls launch on the stream the graph captures
    calls = [st.ctx.prepare_layer_forward(cfg, st.T, p["wr"][l], bias[l], p["slot_of"][l * cfg.E:(l + 1) * cfg.E],
                                          p["n_slots"], p["pool"], p["stride"], p["shared"][l], ws, stream=s)
             for l in range(st.L)]

    def run():
        x = st.x0
        for l, c in enumerate(calls):
            c(x, st.y[l])
            x = st.y[l]

    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = allreduce_max(e0.elapsed_time(e1), world) / steps
    return {"tok_s": round(st.T * world / (ms / 1e3), 1), "layer_us": round(ms * 1e3 / st.L, 3),
            "how": f"{st.L} moe_layer_forward launches per step in one CUDA graph"}


def run_ours(args):
    import torch
    world, rank, local = dist_setup()
    hbm, tf, tf_s, peak_kind = peaks()
    T = args.tokens
    stack_wl = args.workload == "stack"
    pool = make_pool(args.bits, layers=args.layers)
    if stack_wl:  # 256 consecutive decode steps, 7 of each position's 10 experts kept from the step before
        st = DecodeStack(pool, T=T, steps=256, keep=7)
    else:
        st = DecodeStack(pool, T=T)
    steps = args.steps
    ms_max, clocks = time_steps(st, steps, args.warmup, world, local)
    ms_step = ms_max / steps
    scale = LAYERS / st.L  # per 48-layer stack (st.L < 48 only when profiling)
    value = st.T * steps * world / (ms_max / 1e3 * scale)
    rec = stack_record(st, ms_max, steps, args.warmup, hbm, world)
    # roofline of the one kernel of the step: the stack launch's algorithmic
    # bytes over its average duration (CUDA events on its stream)
    idx = [(args.warmup + i) % st.S for i in range(steps)]
    launch_bytes = float(np.mean([st.step_bytes(s) for s in idx]))
    achieved = launch_bytes / (ms_step / 1e3) / 1e9

    # end to end through the public API: pinned host x -> moe_stack_forward ->
    # pinned host y of the last layer, every step inside the timed region
    xh = torch.from_numpy(st.x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty(st.T, st.cfg.d, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.current_stream()
    for i in range(3):
        st.x0.copy_(xh, non_blocking=True)
        yh.copy_(st.step(i)[st.L - 1], non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    n_e2e = max(3, steps // 2)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(n_e2e):
        st.x0.copy_(xh, non_blocking=True)
        yh.copy_(st.step(i)[st.L - 1], non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allreduce_max(e2.elapsed_time(e3), world)
    e2e_value = st.T * n_e2e * world / (e2e_ms / 1e3 * scale)

    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s (48-layer MoE stack)",
        "n_gpus": world,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"u{args.bits} codes x int16 block-requantised activations (dp2a), f32 block sums",
        "data": "synthetic (seeded; random-init weights of the stated shapes)",
        "config": {
            "workload": workload_name(st.T, args.bits, st.L, stack_wl),
            "global_batch": st.T * world, "seq_len": 1, "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2 ({st.L} layers, ~{launch_bytes / 1e9:.2f} GB touched per step)",
            **rec,
        },
        "roofline": {
            "kernel": "decode stack kernel (router, top-k, grouping, experts, combine of all layers), "
                      "one launch per step",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": f"{peak_kind} copy bandwidth",
            "traffic": DECODE_STACK_DRAM_BYTES.get((st.T, args.bits, st.L, stack_wl)),
            "avg_launch_us": round(ms_step * 1e3, 3), "bytes_per_launch": round(launch_bytes),
        },
        "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s (48-layer MoE stack)",
                "h2d_bytes_per_step": st.T * st.cfg.d * 2, "d2h_bytes_per_step": st.T * st.cfg.d * 2,
                "how": "pinned host x -> moe_stack_forward (C ABI) -> pinned host y of the last layer, CUDA events"},
        "gpu_launches": steps,
        "clocks": clocks,
    }
    # the oracle baseline first: the extras free the headline pool
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(st, min(args.cpu_layers, st.L))
    if not args.no_extras and not stack_wl and st.L == LAYERS:
        res["config"]["extras"] = run_extras(args, pool, st, world, local, hbm, tf)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_extras(args, pool2, st1, world, local, hbm, tf):
    """The other configurations, as compact sub-records of the headline line:
    the same layers as 48 single-layer launches; the 48-layer stack at T=4
    over 256 correlated steps; the 3-bit stack at T = 1..4; the T=8192 prefill
    chunk (2- and 3-bit)."""
    import torch
    out = {}
    out["layer_calls_t1"] = layer_call_record(st1, 20, world)
    out["skip_t1_q2"] = skip_record(st1, pool2, skip_from=6)
    st4 = DecodeStack(pool2, T=4, steps=256, keep=7)
    ms, clk = time_steps(st4, 256, 3, world, local)
    out["stack_t4_correlated_q2"] = {**stack_record(st4, ms, 256, 3, hbm, world), "steps": 256, "clocks": clk}
    out["residency_t4_correlated_q2"] = {"stationary": residency_record(st4, pool2)}
    # the same kind of stream with another popularity ranking (a conversation
    # that moved away from the usage the table was seeded with)
    del st4
    st_sh = DecodeStack(pool2, T=4, steps=256, keep=7, seed=SEED + 7)
    out["residency_t4_correlated_q2"]["shifted"] = residency_record(st_sh, pool2)
    del st_sh
    del st1
    torch.cuda.empty_cache()
    for k in ("pool", "shared", "wr"):
        pool2[k] = None
    torch.cuda.empty_cache()
    pool3 = make_pool(3)
    q3 = {}
    for T in (1, 2, 3, 4):
        st3 = DecodeStack(pool3, T=T, steps=64, keep=7)
        ms, _ = time_steps(st3, 64, 3, world, local)
        q3[f"T{T}"] = stack_record(st3, ms, 64, 3, hbm, world)
        del st3
    out["stack_q3_correlated"] = q3
    del pool3
    torch.cuda.empty_cache()
    for bits in (2, 3):
        pl = PrefillLayer(T=8192, bits=bits)
        pl.capture()
        for _ in range(3):
            pl.graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            pl.graph.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = allreduce_max(e0.elapsed_time(e1), world) / 10
        parts = pl.time_parts(reps=3)
        ffn = parts["expert_ffn"]
        ach = pl.flops / (ffn / 1e3) / 1e12
        out[f"prefill_t8192_q{bits}"] = {
            "tok_s_per_layer": round(pl.T * world / (ms / 1e3), 1), "ms_per_layer": round(ms, 4),
            "parts_ms": {k: round(v, 4) for k, v in parts.items()},
            "expert_ffn_tflops": round(ach, 1), "expert_ffn_frac_of_bf16_peak": round(ach / tf, 4),
            "useful_gflop": round(pl.flops / 1e9, 1)}
        del pl
        torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_stack_inputs(st, n_layers):
    """Host copies of the first n_layers layers' inputs (router, bias, slot
    table, shared expert); routed expert records are fetched from the device
    pool when the oracle first asks for one (the fetch time is kept apart)."""
    cfg, p = st.cfg, st.p
    out = []
    for l in range(n_layers):
        wr = p["wr"][l].cpu().numpy()
        bias = st.bias[0, l].cpu().numpy()
        slot_of = p["slot_of"][l * cfg.E:(l + 1) * cfg.E].cpu().numpy()
        out.append((wr, bias, slot_of, p["shared"][l].cpu().numpy()))
    return out


def cpu_baseline(st, n_layers):
    """The fp64 oracle, as it stands, on the first n_layers of the chained
    stack (layer l + 1 reads the oracle's bf16-rounded output of layer l)."""
    from oracle import moe_oracle as O
    cfg, pool = st.cfg, st.p["pool"]
    inputs = oracle_stack_inputs(st, n_layers)
    x = st.x_host
    fetch = [0.0]

    def record(slot_of, e):
        t = time.perf_counter()
        r = pool[int(slot_of[e])].cpu().numpy()
        fetch[0] += time.perf_counter() - t
        return O.sections_from_record(r, cfg.d, cfg.f, cfg.bits)

    t0 = time.perf_counter()
    for wr, bias, slot_of, shared in inputs:
        cache = O.ExpertCache(lambda e, s=slot_of: record(s, e), cfg.d, cfg.f, cfg.bits)
        sh = O.expert_weights(O.sections_from_record(shared, cfg.d, cfg.f, cfg.bits), cfg.d, cfg.f, cfg.bits)
        y = O.layer_forward(x, wr, cfg.k, cache, sh, bias=bias, residual=True)["y"]
        x = _bf16_bits(y)
    dt = time.perf_counter() - t0 - fetch[0]
    per_layer = dt / n_layers
    cores = _oracle_threads()
    return {"value": round(st.T / (per_layer * LAYERS), 4), "unit": "tokens/s (48-layer MoE stack)",
            "cores": cores, "kind": "oracle", "host": cpu_info(),
            "sample": f"first {n_layers} of 48 chained layers at T={st.T} (fp64 numpy oracle, {dt:.1f} s "
                      f"without {fetch[0]:.2f} s of expert-record copies from the device), scaled to 48 layers"}


def _bf16_bits(y):
    """fp64 -> bf16 bits, round to nearest even (the next layer's input)."""
    f = np.asarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((f + 0x7FFF + ((f >> 16) & 1)) >> 16).astype(np.uint16)
    return r


def _oracle_threads():
    import threadpoolctl
    return max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])


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
            "cores": cores, "kind": "oracle", "host": cpu_info(),
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
    cfg_d, cfg_f, E, k, bits = 2048, 768, 512, 10, args.bits
    T = args.tokens
    layers_per_step = 2  # the first two layers of the chain per step
    layers = []
    for l in range(layers_per_step):
        wr = synth.router_weights(E, cfg_d, SEED + 1000 * l + 1)
        bias = synth.bias_from_sets(synth.zipf_sets(T, E, k, SEED + 1000 * l), E)
        sel = np.unique(np.argsort(-bias, axis=1)[:, :k])
        secs = {int(e): synth.expert_sections(cfg_d, cfg_f, bits, SEED + 100 + 1000 * l + int(e)) for e in sel}
        shared = synth.expert_sections(cfg_d, cfg_f, bits, SEED + 99 + 1000 * l)
        layers.append((wr, bias, secs, shared))
    x0 = synth.activations(T, cfg_d, SEED + 16, scale=STACK_X_SCALE)  # as the stack arm's input
    times = []
    for step in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        x = x0
        for wr, bias, secs, shared in layers:
            cache = O.ExpertCache(lambda e, s=secs: s[e], cfg_d, cfg_f, bits)
            sh = O.expert_weights(shared, cfg_d, cfg_f, bits)
            x = _bf16_bits(O.layer_forward(x, wr, k, cache, sh, bias=bias, residual=True)["y"])
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            times.append(dt / layers_per_step)
    per_layer = float(np.mean(times))
    value = T / (per_layer * LAYERS)
    sample = (f"the first {layers_per_step} of 48 chained layers per step at T={T} "
              f"({per_layer * layers_per_step * 1e3:.0f} ms of oracle work per step), scaled to 48 layers")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s (48-layer MoE stack)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_layer * layers_per_step * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(T, bits, correlated=args.workload == "stack"), "global_batch": T,
                   "seq_len": 1, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s (48-layer MoE stack)",
                         "cores": _oracle_threads(), "kind": "oracle", "sample": sample, "host": cpu_info()},
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
    cores = _oracle_threads()
    unit = f"tokens/s (one MoE layer, prefill chunk T={T})"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(float(np.mean(times)) * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"prefill layer d=2048 f=768 E=512 top-10 + 1 shared, T={T}, {bits}-bit "
                               f"(oracle on {n} tokens per step)", "global_batch": n, "seq_len": T,
                   "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 3), "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"{n} of {T} tokens per step", "host": cpu_info()},
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
    ap.add_argument("--no-extras", action="store_true", help="decode: only the headline configuration")
    ap.add_argument("--workload", default="decode", choices=["decode", "stack", "prefill"],
                    help="decode: T tokens, one routing draw; stack: the 48-layer stack over 256 correlated "
                         "decode steps (use --tokens 4 for the verify width); prefill: one layer, T=8192")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="decode: layers in the stack (fewer only to profile a small case)")
    ap.add_argument("--cpu-tokens", type=int, default=32, help="prefill: oracle sample size")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: relaunch under torch.distributed.run
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr=127.0.0.1", "--master-port=29531", os.path.abspath(__file__)] + sys.argv[1:]
        sys.exit(subprocess.call(cmd))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        sys.exit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "prefill":
        run_prefill(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
