"""Benchmark of the quantised MoE decode layer on B200.

One step = one pass of the whole hot path (router, gate/up + SwiGLU, down +
combine + shared expert + residual) for one token of the decode layer
hidden 4096, 512 routed + 1 shared experts, inter 1024, top-10, 4-bit group 64,
through the C ABI (moe_layer_forward).  Weights, router and inputs are seeded
synthetic data generated in HBM.  Steps rotate over 8 layer instances and 16
tokens per instance (128 distinct steps, ~10 GB of distinct expert weights)
so that each step's bytes come from HBM, not L2 (126 MB).

Prints one JSON line (rank 0).  Multi-GPU: independent replicas, one process
per GPU (the decode step of one token does not shard).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantised_expert_ffn_moe_b200 import synth  # noqa: E402

METRIC = "MoE layer µs/token and expert-weight HBM GB/s (% of B200 roofline)"
UNIT = "GB/s"
SHAPE = synth.DECODE_397B
N_INST = 8        # layer instances rotated (default)
N_TOK = 16        # tokens per instance
FALLBACK_HBM = 6650.0

WORKLOADS = {
    4: (synth.DECODE_397B, "decode MoE layer: hidden 4096, 512 routed + 1 shared experts, inter 1024, "
        "top-10 routed + shared, 4-bit affine group 64 (bf16 scale/bias), 1 token per step"),
    2: (synth.DECODE_2BIT, "decode MoE layer: hidden 4096, 512 routed + 1 shared experts, inter 1024, "
        "top-3 routed + shared, 2-bit affine group 64 (bf16 scale/bias), 1 token per step"),
}
WORKLOAD = WORKLOADS[4][1]


def expert_bytes_per_step():
    return (SHAPE.top_k + int(SHAPE.has_shared)) * SHAPE.expert_bytes()


def gateup_bytes_per_step():
    """Gate and up matrices (codes + bf16 scales + biases) of the k routed
    experts and the shared one: what the gate/up kernel must read."""
    n = SHAPE.hidden * SHAPE.inter
    per_mat = n * SHAPE.bits // 8 + 2 * 2 * n // SHAPE.group
    return (SHAPE.top_k + int(SHAPE.has_shared)) * 2 * per_mat


def router_bytes():
    return SHAPE.n_experts * SHAPE.hidden * 2


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM, "fallback"


# the sources the decode kernels (k_route, k_gateup, k_down) are built from
DECODE_SOURCES = ("common.cuh", "image.cuh", "route.cuh", "ffn.cuh")


def measured_tensor_peak():
    """Dense bf16 tensor TFLOP/s (burst) of MEASURED_PEAKS.json; fp16 MMAs
    have the same dense rate."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantised_expert_ffn_moe_b200", "csrc")
    for f in DECODE_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch recorded from an ncu capture, valid only while
    the kernel sources are unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d.get("k_gateup_dram_bytes_per_launch", {}).get(str(SHAPE.bits))


class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix="moeq_clocks_", suffix=".csv")
        os.close(fd)

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.remove(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The maximum of v over the ranks (every rank gets it); NCCL on the GPU,
    gloo on the CPU."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


# ------------------------------------------------------------------ oracle --

def oracle_rate(seconds_min=10.0, max_tokens=8, seed=0):
    """The CPU oracle (single-threaded C, fp64) on whole layer-tokens of the
    same workload: expert-weight GB/s and the sample description."""
    import oracle as orc
    lay = synth.make_layer(SHAPE, seed, "cpu")
    xs = synth.make_tokens(SHAPE, max_tokens, seed, "cpu")
    xb = synth.to_np_bits(xs)
    wr = synth.to_np_bits(lay.router)
    sg = synth.to_np_bits(lay.shared_gate)

    def hexp(e):
        m = lay.experts.mats(e)
        return orc.Expert(*[tuple(synth.to_np_bits(a) for a in m[k]) for k in ("gate", "up", "down")])

    shared = hexp(SHAPE.n_experts)
    done, t_total = 0, 0.0
    while done < max_tokens and (t_total < seconds_min or done < 2):
        x = xb[done:done + 1]
        _, idx, _ = orc.route(orc.bf16_to_f64(x[0]), wr, SHAPE.top_k)
        experts = {int(e): hexp(int(e)) for e in idx}
        t0 = time.perf_counter()
        orc.layer_forward(SHAPE.desc(), x, x, wr, experts, shared, sg)
        t_total += time.perf_counter() - t0
        done += 1
    gbs = done * expert_bytes_per_step() / t_total / 1e9
    sample = (f"{done} whole layer-tokens of this workload (router + {SHAPE.top_k + 1} expert FFNs + combine), "
              f"fp64 C oracle")
    return gbs, done, t_total, sample


def run_reference(args, rank, world):
    if rank != 0:
        return
    # each step: the oracle's quantised mat-vec over a slice of one selected
    # expert's matrices, sized so warm-up + steps stay within ~60 s
    import oracle as orc
    lay_experts = synth.make_experts(SHAPE, 0, "cpu", n=3)
    mats = []
    for e in range(3):
        m = lay_experts.mats(e)
        for k, cols in (("gate", SHAPE.hidden), ("up", SHAPE.hidden), ("down", SHAPE.inter)):
            mats.append((tuple(synth.to_np_bits(a) for a in m[k]), cols))
    budget = 60.0 / max(1, args.steps + args.warmup)
    # calibrate: seconds per row of a gate matrix
    (c, s, b), cols = mats[0]
    xv = np.random.default_rng(0).normal(0, 1, cols)
    t0 = time.perf_counter()
    orc.qmatvec(SHAPE.bits, 64, c[:16], s[:16], b[:16], xv)
    per_row = (time.perf_counter() - t0) / 16
    rows = int(max(16, min(1024, budget / max(per_row, 1e-9))) // 16 * 16)
    bytes_done, t_total = 0, 0.0
    for i in range(args.warmup + args.steps):
        (c, s, b), cols = mats[i % len(mats)]
        r0 = (i * rows) % (c.shape[0] - rows + 1)
        xv = np.random.default_rng(i).normal(0, 1, cols)
        t0 = time.perf_counter()
        orc.qmatvec(SHAPE.bits, 64, c[r0:r0 + rows], s[r0:r0 + rows], b[r0:r0 + rows], xv)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            t_total += dt
            bytes_done += rows * (cols * SHAPE.bits // 8 + cols // 64 * 4)
    value = bytes_done / t_total / 1e9
    sample = (f"each step: the oracle's fp64 quantised mat-vec (materialise W, then dot) over "
              f"{rows} rows of one expert matrix of this workload")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_total / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": sample, "value": value, "unit": UNIT},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- GPU ---

def run_gpu(args, rank, world, local):
    from quantised_expert_ffn_moe_b200 import moeq
    N_INST = args.instances
    dev = torch.device("cuda", local)
    torch.manual_seed(1234 + rank)
    stream = torch.cuda.current_stream()
    desc = moeq.make_desc(SHAPE)
    layers, slots, xs = [], [], []
    for i in range(N_INST):
        lay = synth.make_layer(SHAPE, 1000 * rank + i, dev)
        layers.append(lay)
        slots.append(moeq.DeviceSlots(lay.experts, SHAPE.n_experts))
        xs.append(synth.make_tokens(SHAPE, N_TOK, 50 + 1000 * rank + i, dev))
    outs = [torch.empty_like(x) for x in xs]
    ws = moeq.workspace(desc, 1, dev)
    G = N_INST * N_TOK

    def step(j):
        i, t = j % N_INST, (j // N_INST) % N_TOK
        moeq.layer_forward(desc, xs[i][t:t + 1], xs[i][t:t + 1], layers[i].router, slots[i], ws,
                           shared_gate=layers[i].shared_gate, out=outs[i][t:t + 1], stream=stream)

    # warm-up (also does the library's one-time per-device set-up)
    for j in range(max(args.warmup, 3)):
        step(j)
    torch.cuda.synchronize()

    def capture(n):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for j in range(n):
                    i, t = j % N_INST, (j // N_INST) % N_TOK
                    moeq.layer_forward(desc, xs[i][t:t + 1], xs[i][t:t + 1], layers[i].router,
                                       slots[i], ws, shared_gate=layers[i].shared_gate,
                                       out=outs[i][t:t + 1], stream=s)
        torch.cuda.current_stream().wait_stream(s)
        return g

    full, tail = args.steps // G, args.steps % G
    g_full = capture(G) if full else None
    g_tail = capture(tail) if tail else None
    # graph warm-up
    for _ in range(max(1, args.warmup // G)):
        if g_full:
            g_full.replay()
        elif g_tail:
            g_tail.replay()
    torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record()
        for _ in range(full):
            g_full.replay()
        if g_tail:
            g_tail.replay()
        ev1.record()
        torch.cuda.synchronize()
        barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, world)
    clocks = clk.summary()
    sec = ms / 1e3
    us_tok = sec / args.steps * 1e6
    eb = expert_bytes_per_step()
    gu_bytes, dn_bytes = gateup_bytes_per_step(), eb - gateup_bytes_per_step()
    value = world * args.steps * eb / sec / 1e9   # whole-job expert-weight GB/s
    per_gpu = args.steps * eb / sec / 1e9
    peak, peak_kind = measured_peaks()

    # end to end through the public API with host buffers (pinned), eager
    e2e_steps = min(args.steps, args.e2e_steps)
    xh = torch.empty((e2e_steps, SHAPE.hidden), dtype=torch.bfloat16).pin_memory()
    xh.copy_(xs[0].cpu().repeat((e2e_steps + N_TOK - 1) // N_TOK, 1)[:e2e_steps])
    oh = torch.empty_like(xh).pin_memory()
    xd = [torch.empty((1, SHAPE.hidden), dtype=torch.bfloat16, device=dev) for _ in range(N_INST)]
    od = [torch.empty_like(x) for x in xd]
    for j in range(3):
        i = j % N_INST
        xd[i].copy_(xh[j:j + 1], non_blocking=True)
        moeq.layer_forward(desc, xd[i], xd[i], layers[i].router, slots[i], ws,
                           shared_gate=layers[i].shared_gate, out=od[i])
        oh[j:j + 1].copy_(od[i], non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    ev0.record()
    for j in range(e2e_steps):
        i = j % N_INST
        xd[i].copy_(xh[j:j + 1], non_blocking=True)
        moeq.layer_forward(desc, xd[i], xd[i], layers[i].router, slots[i], ws,
                           shared_gate=layers[i].shared_gate, out=od[i])
        oh[j:j + 1].copy_(od[i], non_blocking=True)
    ev1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    e2e_value = world * e2e_steps * eb / (e2e_ms / 1e3) / 1e9
    # per-kernel device time: events between the layer's three kernels
    # (router | gate/up + SwiGLU | down + combine), on the launching stream,
    # averaged over KT calls after the timed region
    KT = 256
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(KT)]
    for es in evs:
        for e in es:
            e.record(stream)  # creates the handle
    torch.cuda.synchronize()
    for j in range(KT):
        moeq.set_kernel_events(evs[j])
        step(j)
    moeq.set_kernel_events(None)
    torch.cuda.synchronize()
    kern_ms = [sum(evs[j][q].elapsed_time(evs[j][q + 1]) for j in range(KT)) / KT for q in range(3)]
    kern_ms = [max_over_ranks(v, world) for v in kern_ms]
    rc, st = moeq.device_status(ws)
    if rc != 0:
        raise SystemExit(f"device status {st:#x} after the timed region")

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        gbs, n_tok, t_cpu, sample = oracle_rate()
        cpu = {"value": gbs, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
               "seconds": t_cpu, "us_per_token": t_cpu / n_tok * 1e6}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": f"u{SHAPE.bits} codes x 16-bit fixed-point activations, int8 MMA int32 accumulate, fp32 epilogue",
        "data": "synthetic (seeded; random codes, U(0.005,0.02) scales, U(-0.08,0.08) biases, N(0,0.02) router)",
        "us_per_token": us_tok,
        "expert_bytes_per_token": eb,
        "router_bytes_per_token": router_bytes(),
        "config": {"workload": WORKLOAD, "global_batch": world, "tokens_per_step_per_gpu": 1,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: steps rotate over 8 layer instances x 16 tokens "
                         "(128 distinct steps, ~10 GB of expert weights between reuses of a step's data)",
                   "graph": "K steps replayed from CUDA graphs of 128 layer calls"},
        "roofline": {"bound": "hbm", "achieved": gu_bytes / (kern_ms[1] / 1e3) / 1e9, "peak": peak,
                     "unit": "GB/s", "frac": gu_bytes / (kern_ms[1] / 1e3) / 1e9 / peak,
                     "peak_kind": f"{peak_kind} (copy GB/s)",
                     "kernel": "k_gateup (gate/up dequant mat-vecs + SwiGLU, routing top-k in its prologue)",
                     "algorithmic_bytes_per_launch": gu_bytes,
                     "launch_us": kern_ms[1] * 1e3, "launches_timed": KT,
                     "traffic": recorded_traffic()},
        "kernels_us": {"k_route": kern_ms[0] * 1e3, "k_gateup": kern_ms[1] * 1e3, "k_down": kern_ms[2] * 1e3,
                       "k_down_bytes_per_launch": dn_bytes, "k_route_bytes_per_launch": router_bytes()},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "steps": e2e_steps,
                "h2d_bytes_per_step": SHAPE.hidden * 2, "d2h_bytes_per_step": SHAPE.hidden * 2},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


PREFILL_T = 512
PREFILL_WORKLOAD = ("prefill MoE layer: 512 tokens x hidden 4096, 512 routed + 1 shared experts, inter 1024, "
                    "top-10 routed + shared, 4-bit affine group 64, Zipf(1.1)-skewed routing; expert-sorted "
                    "dequant-fused GEMMs on tcgen05")


def run_prefill(args, rank, world, local):
    """The 512-token prefill layer: one layer call of 512 tokens per step,
    rotating over layer instances; value = bytes of the distinct experts a
    step reads / device time (whole job)."""
    from quantised_expert_ffn_moe_b200 import moeq
    n_inst = max(1, min(args.instances, 8))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    desc = moeq.make_desc(SHAPE)
    T, k = PREFILL_T, SHAPE.top_k
    layers, slots, xs, biases = [], [], [], []
    for i in range(n_inst):
        lay = synth.make_layer(SHAPE, 2000 * rank + i, dev)
        layers.append(lay)
        slots.append(moeq.DeviceSlots(lay.experts, SHAPE.n_experts))
        xs.append(synth.make_tokens(SHAPE, T, 70 + 1000 * rank + i, dev))
        biases.append(torch.tensor(synth.zipf_logit_bias(SHAPE.n_experts, T, 1.1, 9 + i), device=dev))
    ws = moeq.workspace(desc, T, dev)
    outs = [torch.empty_like(x) for x in xs]
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)

    def step(j, topk=None):
        i = j % n_inst
        moeq.layer_forward(desc, xs[i], xs[i], layers[i].router, slots[i], ws, shared_gate=layers[i].shared_gate,
                           logit_bias=biases[i], out=outs[i], topk_idx=topk, stream=stream)

    n = SHAPE.hidden * SHAPE.inter
    per_mat = n * SHAPE.bits // 8 + 2 * 2 * n // SHAPE.group
    distinct, pairs = [], T * (k + int(SHAPE.has_shared))
    for i in range(n_inst):
        step(i, topk=idx)
        distinct.append(len(torch.unique(idx)) + int(SHAPE.has_shared))
    for j in range(max(args.warmup, 3)):
        step(j)
    torch.cuda.synchronize()
    steps = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record()
        for j in range(steps):
            step(j)
        ev1.record()
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    sec = ms / 1e3
    wbytes = sum(distinct[j % n_inst] for j in range(steps)) * 3 * per_mat
    value = world * wbytes / sec / 1e9
    per_gpu = wbytes / sec / 1e9
    flops = steps * pairs * 3 * 2 * n
    # per-kernel device time with events between the kernels (router |
    # sort + gate/up GEMM | down GEMM + combine)
    KT = 16
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(KT)]
    for es in evs:
        for e in es:
            e.record(stream)
    torch.cuda.synchronize()
    for j in range(KT):
        moeq.set_kernel_events(evs[j])
        step(j)
    moeq.set_kernel_events(None)
    torch.cuda.synchronize()
    kern_ms = [max_over_ranks(sum(evs[j][q].elapsed_time(evs[j][q + 1]) for j in range(KT)) / KT, world)
               for q in range(3)]
    gu_bytes = sum(distinct[j % n_inst] for j in range(KT)) / KT * 2 * per_mat
    peak, peak_kind = measured_peaks()
    tpeak, tpeak_kind = measured_tensor_peak()
    gemm_tflops = pairs * 3 * 2 * n / ((kern_ms[1] + kern_ms[2]) / 1e3) / 1e12
    # end to end: tokens from pinned host memory, output back, eager
    e2e_steps = min(steps, 32)
    xh = xs[0].cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(xs[0])
    torch.cuda.synchronize()
    barrier(world)
    ev0.record()
    for j in range(e2e_steps):
        i = j % n_inst
        xd.copy_(xh, non_blocking=True)
        moeq.layer_forward(desc, xd, xd, layers[i].router, slots[i], ws, shared_gate=layers[i].shared_gate,
                           logit_bias=biases[i], out=outs[i], stream=stream)
        oh.copy_(outs[i], non_blocking=True)
    ev1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    e2e_bytes = sum(distinct[j % n_inst] for j in range(e2e_steps)) * 3 * per_mat
    rc, st = moeq.device_status(ws)
    if rc != 0:
        raise SystemExit(f"device status {st:#x} after the timed region")
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u4 codes dequantised to fp16, fp16 x fp16 tcgen05 MMA, fp32 accumulate",
        "data": "synthetic (seeded; random codes, U(0.005,0.02) scales, U(-0.08,0.08) biases, N(0,0.02) router, "
                "Zipf(1.1) routing skew through the logit bias)",
        "us_per_token": ms / steps / T * 1e3,
        "expert_bytes_per_step": wbytes / steps,
        "distinct_experts_per_step": sum(distinct) / n_inst,
        "tensor_tflops": flops / sec / 1e12,
        "config": {"workload": PREFILL_WORKLOAD, "global_batch": world * T, "tokens_per_step_per_gpu": T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"inputs larger than L2: each step reads ~{wbytes / steps / 1e9:.1f} GB of expert weights "
                         f"(L2 126 MB), {n_inst} layer instances rotated"},
        "roofline": {"bound": "hbm", "achieved": gu_bytes / (kern_ms[1] / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": gu_bytes / (kern_ms[1] / 1e3) / 1e9 / peak, "peak_kind": f"{peak_kind} (copy GB/s)",
                     "kernel": "pair sort + k_pf_gateup (gate/up GEMM + SwiGLU on tcgen05)",
                     "algorithmic_bytes_per_launch": gu_bytes, "launch_us": kern_ms[1] * 1e3,
                     "launches_timed": KT, "traffic": None},
        "kernels_us": {"k_route": kern_ms[0] * 1e3, "sort_and_k_pf_gateup": kern_ms[1] * 1e3,
                       "k_pf_down_and_combine": kern_ms[2] * 1e3},
        "tensor_roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": tpeak, "unit": "TFLOP/s",
                            "frac": gemm_tflops / tpeak,
                            "peak_kind": f"{tpeak_kind} dense bf16 (fp16 MMAs have the same rate)",
                            "kernels": "pair sort + k_pf_gateup + k_pf_down + combine",
                            "flop_per_launch": pairs * 3 * 2 * n},
        "cpu_baseline": None,
        "e2e": {"value": world * e2e_bytes / (e2e_ms / 1e3) / 1e9, "unit": UNIT, "steps": e2e_steps,
                "h2d_bytes_per_step": T * SHAPE.hidden * 2, "d2h_bytes_per_step": T * SHAPE.hidden * 2},
        "gpu_launches": 8 * steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        gbs, n_tok, t_cpu, sample = oracle_rate(max_tokens=2)
        line["cpu_baseline"] = {"value": gbs, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                                "seconds": t_cpu, "us_per_token": t_cpu / n_tok * 1e6}
    print(json.dumps(line), flush=True)


STACK_LAYERS = 16
STACK_TOKENS = 64
STACK_REPEAT = 0.27
STACK_WORKLOAD = ("decode stack: 16 sequential MoE layers of the hidden 4096, 512 routed + 1 shared, inter 1024, "
                  "top-10, 4-bit group 64 shape (~58 GB of expert weights resident), RMS normalisation before each "
                  "layer, one token chained layer to layer through the residual, 64-token decode loop whose expert "
                  "sets repeat 27% between consecutive tokens")


def run_stack(args, rank, world, local):
    """One step = one token through the 16-layer stack (normalise, route,
    experts, combine into the residual, per layer); the 64 tokens of the loop
    are replayed from one CUDA graph."""
    from quantised_expert_ffn_moe_b200 import moeq
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    desc = moeq.make_desc(SHAPE)
    L, T, E, k = STACK_LAYERS, STACK_TOKENS, SHAPE.n_experts, SHAPE.top_k
    layers, slots, biases = [], [], []
    for l in range(L):
        lay = synth.make_layer(SHAPE, 3000 * rank + l, dev)
        layers.append(lay)
        slots.append(moeq.DeviceSlots(lay.experts, E))
        b, _ = synth.repeat_logit_bias(E, k, T, STACK_REPEAT, 40 + l)
        biases.append(torch.tensor(b, device=dev))
    xs = synth.make_tokens(SHAPE, T, 90 + 1000 * rank, dev)
    hs = torch.empty_like(xs)     # each token's final hidden state
    ws = moeq.workspace(desc, 1, dev)

    def token(t, s):
        # layer 0 reads the token's input and writes its state; later layers
        # update the state in place
        h = hs[t:t + 1]
        for l in range(L):
            src = xs[t:t + 1] if l == 0 else h
            moeq.layer_forward_normed(desc, src, layers[l].router, slots[l], ws, 1e-6,
                                      shared_gate=layers[l].shared_gate, logit_bias=biases[l][t:t + 1], out=h,
                                      stream=s)

    for t in range(max(args.warmup, 3)):
        token(t % T, stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            for t in range(T):
                token(t, cs)
    torch.cuda.current_stream().wait_stream(cs)
    loops = max(1, (args.steps + T - 1) // T)
    steps = loops * T
    g.replay()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record()
        for _ in range(loops):
            g.replay()
        ev1.record()
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    sec = ms / 1e3
    eb = expert_bytes_per_step()           # per layer-token
    value = world * steps * L * eb / sec / 1e9
    # per-kernel device time over the layer calls of the first KT // L tokens
    # (eager), which also records their routing
    KT = 256
    TK = KT // L
    idx = torch.empty((TK, L, k), dtype=torch.int32, device=dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(KT)]
    for es in evs:
        for e in es:
            e.record(stream)
    torch.cuda.synchronize()
    for t in range(TK):
        h = hs[t:t + 1]
        for l in range(L):
            src = xs[t:t + 1] if l == 0 else h
            moeq.set_kernel_events(evs[t * L + l])
            moeq.layer_forward_normed(desc, src, layers[l].router, slots[l], ws, 1e-6,
                                      shared_gate=layers[l].shared_gate, logit_bias=biases[l][t:t + 1], out=h,
                                      topk_idx=idx[t, l:l + 1], stream=stream)
            moeq.set_kernel_events(None)
    torch.cuda.synchronize()
    kern_ms = [max_over_ranks(sum(evs[i][q].elapsed_time(evs[i][q + 1]) for i in range(KT)) / KT, world)
               for q in range(3)]
    ia = idx.cpu().numpy()
    reuse = float(np.mean([len(set(ia[t, l]) & set(ia[t - 1, l])) / k for t in range(1, TK) for l in range(L)]))
    gu_bytes = gateup_bytes_per_step()
    peak, peak_kind = measured_peaks()
    # end to end: each token's input from pinned host memory, its final
    # hidden state back, eager calls through the public API
    e2e_steps = min(steps, 2 * T)
    xh = xs.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    hd = torch.empty((1, SHAPE.hidden), dtype=torch.bfloat16, device=dev)
    spec = [(desc, layers[l].router, slots[l], layers[l].shared_gate) for l in range(L)]
    torch.cuda.synchronize()
    barrier(world)
    ev0.record()
    for j in range(e2e_steps):
        t = j % T
        hd.copy_(xh[t:t + 1], non_blocking=True)
        moeq.stack_forward(spec, hd, ws, 1e-6, [b[t:t + 1] for b in biases], stream=stream)
        oh[t:t + 1].copy_(hd, non_blocking=True)
    ev1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    rc, st = moeq.device_status(ws)
    if rc != 0:
        raise SystemExit(f"device status {st:#x} after the timed region")
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u4 codes x 16-bit fixed-point activations, int8 MMA int32 accumulate, fp32 epilogue",
        "data": "synthetic (seeded; random codes, U(0.005,0.02) scales, U(-0.08,0.08) biases, N(0,0.02) router, "
                "27%-repeat routing through the logit bias)",
        "us_per_layer_token": ms / steps / L * 1e3,
        "us_per_token": ms / steps * 1e3,
        "expert_bytes_per_step": L * eb,
        "expert_reuse_between_tokens": reuse,
        "config": {"workload": STACK_WORKLOAD, "global_batch": world, "tokens_per_step_per_gpu": 1,
                   "layers": L, "loop_tokens": T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: ~1.2 GB of expert weights per token across the 16 layers "
                         "(L2 126 MB) between two visits of a layer",
                   "graph": "the 64-token loop (16 layers x 3 kernels per token; the normalisation runs inside "
                            "the router kernel) as one CUDA graph"},
        "roofline": {"bound": "hbm", "achieved": gu_bytes / (kern_ms[1] / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": gu_bytes / (kern_ms[1] / 1e3) / 1e9 / peak, "peak_kind": f"{peak_kind} (copy GB/s)",
                     "kernel": "k_gateup (gate/up dequant mat-vecs + SwiGLU, routing top-k in its prologue)",
                     "algorithmic_bytes_per_launch": gu_bytes, "launch_us": kern_ms[1] * 1e3,
                     "launches_timed": KT, "traffic": recorded_traffic()},
        "kernels_us": {"k_route": kern_ms[0] * 1e3, "k_gateup": kern_ms[1] * 1e3, "k_down": kern_ms[2] * 1e3},
        "cpu_baseline": None,
        "e2e": {"value": world * e2e_steps * L * eb / (e2e_ms / 1e3) / 1e9, "unit": UNIT, "steps": e2e_steps,
                "h2d_bytes_per_step": SHAPE.hidden * 2, "d2h_bytes_per_step": SHAPE.hidden * 2},
        "gpu_launches": 3 * L * steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        gbs, n_tok, t_cpu, sample = oracle_rate(max_tokens=4)
        line["cpu_baseline"] = {"value": gbs, "unit": UNIT, "cores": 1, "kind": "oracle",
                                "sample": sample + " (one layer of the stack)",
                                "seconds": t_cpu, "us_per_token": t_cpu / n_tok * 1e6}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=256)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bits", type=int, default=4, choices=[4, 2],
                    help="4: the top-10 + shared 4-bit decode layer (default); 2: the 2-bit top-3 + shared layer")
    ap.add_argument("--prefill", action="store_true",
                    help="the 512-token prefill layer (4-bit) instead of one decode token per step")
    ap.add_argument("--stack", action="store_true",
                    help="the 16-layer decode stack (4-bit), one token through all layers per step")
    ap.add_argument("--instances", type=int, default=N_INST,
                    help="layer instances rotated (fewer only for small profiling runs)")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    global SHAPE, WORKLOAD
    SHAPE, WORKLOAD = WORKLOADS[args.bits]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.prefill:
            if args.steps == 20000:
                args.steps = 200
            if args.warmup == 256:
                args.warmup = 5
            run_prefill(args, rank, world, local)
        elif args.stack:
            if args.steps == 20000:
                args.steps = 640
            if args.warmup == 256:
                args.warmup = 64
            run_stack(args, rank, world, local)
        else:
            run_gpu(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
