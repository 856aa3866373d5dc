"""Benchmark of the affine-quantised MoE FFN layer on B200.

One JSON line on rank 0.  A step is one forward of the whole layer (router
qmv, routing, gate/up + SwiGLU, down, combine) for the workload's batch of
tokens.  Default workload: single-token decode of the 4096-hidden,
512-expert, top-4, 4-bit layer with a 4-bit shared expert and 8-bit router
and sigmoid gate.  Inputs are seeded synthetic weights and activations.

L2: the timed steps cycle through `--copies` independent copies of the
layer (router, shared expert and expert bank each) with a fresh token per
step, so the bytes touched between two uses of any weight exceed the 126 MB
L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own replica on its own tokens (the
decode path does not shard); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (shape, tokens per step)
    "decode_397b_m1": ("decode_397b", 1),
    # same shapes with a 16-expert bank: small enough for full ncu captures
    "decode_397b_e16_m1": ("decode_397b_e16", 1),
    "decode_397b_e64_m8": ("decode_397b_e64", 8),
    "tiny_m1": ("tiny", 1),
    "tiny_m3": ("tiny", 3),
    "tiny_m5": ("tiny", 5),
    "decode_397b_m8": ("decode_397b", 8),
    "decode_397b_m64": ("decode_397b", 64),
    "decode_30b_m1": ("decode_30b", 1),
    "decode_mixed_2bit_m1": ("mixed_2bit", 1),
    # prefill: one call over M tokens per step
    "prefill_8bit_m16032": ("prefill_8bit", 16032),
    "prefill_8bit_m16068": ("prefill_8bit", 16068),
    "prefill_8bit_m16384": ("prefill_8bit", 16384),
    "prefill_mixed_2bit_m256": ("mixed_2bit", 256),
    "prefill_mixed_2bit_m4096": ("mixed_2bit", 4096),
    # small prefill case for full profiler captures
    "prefill_8bit_m2048": ("prefill_8bit", 2048),
}
METRIC = "qMoE layer tokens/s"


def shape(name):
    """Layer shape by name (plain data: loads no library)."""
    import dataclasses
    from quantized_mixture_experts_affine_b200.config import CONFIGS
    if name in ("decode_397b_e16", "decode_397b_e64"):
        return dataclasses.replace(CONFIGS["decode_397b"], name=name, E=int(name[-2:]))
    return CONFIGS[name]


def config_of(workload, world, copies):
    """The line's `config`: the workload's shape and how the timed steps
    keep their weights out of L2 (the same dict in both arms)."""
    cfg_name, M = WORKLOADS[workload]
    cfg = shape(cfg_name)
    d = {"workload": workload, "tokens_per_step": M, "hidden": cfg.H, "experts": cfg.E,
         "top_k": cfg.K, "intermediate": cfg.I, "expert_bits": cfg.expert_bits,
         "router_bits": cfg.router_bits, "shared_expert": cfg.shared,
         "shared_intermediate": cfg.shared_I, "group_size": cfg.G,
         "parallelism": f"replicas{world}"}
    if workload.startswith("prefill"):
        d["l2"] = "inputs larger than L2 (weights, token rows and output rows)"
    else:
        touched = (cfg.router_bytes() + min(cfg.E, M * cfg.K) * cfg.expert_bytes()
                   + cfg.shared_bytes())
        mb = copies * touched / 1e6
        d["l2"] = (f"{copies} layer copies cycled, fresh tokens per step (up to {mb:.0f} MB "
                   f"of weights touched per cycle; L2 is 126 MB"
                   + (", so these weights stay L2-resident)" if mb < 126 else ")"))
    return d
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# kernel each roofline line names, from one ncu capture of the current
# kernels on that workload: decode gate/up launch (it also carries the down
# projections' L2 prefetch), prefill gate/up gather-QMM.  Other workloads:
# not captured (null).
TRAFFIC = {
    "decode_397b_m1": 33131776 + 0,
    "prefill_8bit_m16068": 959738624 + 185099264,
}


def gateup_kernel(cfg, M):
    """Name of the decode gate/up launch the library runs for this layer and
    token count: one token of 2-, 4- or 8-bit affine experts (a shared expert
    of the same width, or 4-bit beside 2-bit experts) behind an 8-bit router
    with at most 512 experts runs on the single-token launches (their
    shared-memory limit aside); everything else on the general GEMV."""
    bs = cfg.shared_bits if cfg.shared else cfg.expert_bits
    single = (M == 1 and cfg.expert_bits in (2, 4, 8) and cfg.router_bits == 8
              and cfg.E <= 512 and cfg.K <= 16
              and (bs == cfg.expert_bits or (cfg.expert_bits, bs) == (2, 4))
              and os.environ.get("MOEQ_SINGLE_DECODE") != "0")
    return ("k_s1_gateup (top-K + gate/up + SwiGLU, single token)" if single
            else "k_gemv gate/up+SwiGLU")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_397b_m1", choices=sorted(WORKLOADS))
    ap.add_argument("--copies", type=int, default=8)
    ap.add_argument("--cpu-sample", type=int, default=8,
                    help="tokens of the bounded oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the secondary prefill measurement of the decode run")
    ap.add_argument("--prefill-workload", default="prefill_8bit_m16068")
    ap.add_argument("--sweep", action="store_true",
                    help="per-config table instead of the benchmark line (one JSON line per row)")
    ap.add_argument("--sweep-rows", default="", help="comma-separated rows (C1..C5) to run")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
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
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML (read-only) every
    ~1 ms from a background thread for the duration of the timed region."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.err = None
        self._stop = False
        self._thread = None

    def _sample(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        self.samples.append((sm, r))

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            dev = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.gpu
            if dev:
                ids = [d for d in dev.split(",") if d.strip()]
                if self.gpu < len(ids) and ids[self.gpu].strip().isdigit():
                    idx = int(ids[self.gpu])
            h = nv.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._sample(nv, h)
            self._ready = True
            while not self._stop:
                time.sleep(0.001)
                self._sample(nv, h)
            self._sample(nv, h)
            nv.nvmlShutdown()
        except Exception as e:  # no NVML: report it, never guess
            self.err = repr(e)
            self._ready = True

    def __enter__(self):
        import threading
        self._ready = False
        self.max_mhz = None
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        t0 = time.time()
        while not self._ready and time.time() - t0 < 10:
            time.sleep(0.001)
        return self

    def __exit__(self, *a):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=10)

    def summary(self):
        if self.err or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": [f"clock sampling unavailable: {self.err}"]}
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "source": "NVML, ~1 ms period, during the timed region"}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def sustained_bf16_peak():
    """The bf16 dense peak for work timed inside a long run (the power cap
    holds the clocks below their burst level): the measured sustained figure,
    else the recipe's fallback of 1.4 PFLOP/s."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops_sustained" in d:
            return d["bf16_tflops_sustained"], "measured sustained"
    return 1400.0, "fallback sustained"


# ------------------------------------------------------------------ CPU oracle sample
class OracleSample:
    """The oracle as it stands, on a bounded sample of the workload: n_tokens
    tokens with their router, routed experts and shared expert generated on
    the host once (not timed).  run(tokens) times the oracle's router qmv,
    routing and experts + combine for those tokens on all host cores."""

    def __init__(self, cfg, n_tokens, seed=0):
        import numpy as np
        import oracle
        from oracle.synthetic import host_router, oracle_layer
        from quantized_mixture_experts_affine_b200 import synth
        self.cfg, self.oracle, self.np = cfg, oracle, np
        self.xb = synth.normal_bf16_host(seed, synth.tag(synth.X, 9999),
                                         n_tokens * cfg.H).reshape(n_tokens, cfg.H)
        self.R = host_router(cfg, seed, 0)
        logits = oracle.qmv(self.R, self.xb)
        idx, self.w, _ = oracle.route(logits, cfg.K, cfg.renorm, cfg.router_scale)
        experts = np.unique(idx)
        self.L = oracle_layer(cfg, seed, 0, experts)
        remap = {int(e): i for i, e in enumerate(experts)}
        self.idx_c = np.vectorize(lambda e: remap[int(e)])(idx).astype(np.int32)
        self.threads = oracle.get_threads()

    def cores(self, n_rows):
        """Threads the oracle actually uses for n_rows tokens (it splits tokens)."""
        return min(self.threads, n_rows)

    def run(self, rows, threads=None):
        """Seconds of the oracle on the sample's tokens `rows` (threads: all
        host cores when None)."""
        o, c = self.oracle, self.cfg
        prev = o.get_threads()
        if threads is not None:
            o.set_threads(threads)
        try:
            x = self.xb[rows]
            t0 = time.perf_counter()
            logits = o.qmv(self.R, x)
            o.route(logits, c.K, c.renorm, c.router_scale)
            o.expert_ffn(self.L, x, self.idx_c[rows], self.w[rows])
            return time.perf_counter() - t0
        finally:
            o.set_threads(prev)


# ------------------------------------------------------------------ reference arm (the oracle)
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg_name, M = WORKLOADS[args.workload]
    cfg = shape(cfg_name)
    pool = max(M, min(args.cpu_sample, args.steps * M))
    smp = OracleSample(cfg, pool)
    for w in range(args.warmup):
        smp.run(list(range(w * M % pool, w * M % pool + M)) if pool >= M else list(range(M)))
        if w >= 2:
            break
    total = 0.0
    for s in range(args.steps):
        r0 = (s * M) % (pool - M + 1)
        total += smp.run(list(range(r0, r0 + M)))
    value = M * args.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(args.workload, args.gpus, args.copies),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": smp.cores(M),
                             "kind": "oracle",
                             "sample": f"{args.steps} steps of {M} token(s) of {args.workload}, "
                                       f"drawn from a pool of {pool} tokens"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ prefill measurement
def layer_flop_of(workload):
    cfg_name, M = WORKLOADS[workload]
    return M * shape(cfg_name).flops_per_token()


def timed_replays(fn, reps, st, world, local):
    """Device time (max over ranks, ms) of reps calls of fn on stream st,
    bracketed by a barrier and a synchronize, with the SM clocks sampled."""
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(st):
            e0.record(st)
            for _ in range(reps):
                fn()
            e1.record(st)
        st.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(e0.elapsed_time(e1), world), clk


def measure_prefill(workload, steps, warmup, world, seed, want_e2e=True, min_ms=100):
    """Timed one-shot prefill calls of `workload` (M tokens each): device
    throughput, the gate/up gather-QMM duration per launch (events around it
    inside captured graphs), tensor-core roofline and end-to-end rate."""
    import torch
    from quantized_mixture_experts_affine_b200 import moeq, synth
    from quantized_mixture_experts_affine_b200.layer import Workspace, synthetic_layer
    cfg_name, M = WORKLOADS[workload]
    cfg = shape(cfg_name)
    L = synthetic_layer(cfg, seed, 0)
    n_x = 2
    xs = synth.normal_bf16_dev(seed, synth.tag(synth.X, 555), n_x * M * cfg.H).view(n_x, M, cfg.H)
    y = torch.empty((M, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((M, cfg.K), dtype=torch.int32, device="cuda")
    w = torch.empty((M, cfg.K), dtype=torch.float32, device="cuda")
    ws = Workspace(L, M, moeq.MODE_PREFILL)
    st = torch.cuda.Stream()
    # the weights and tokens are drawn on the current stream: done before st uses them
    torch.cuda.synchronize()

    def step(i):
        moeq.moeq_layer_forward(L.desc, xs[i % n_x], M, y, None, idx, w, ws.buf, ws.bytes,
                                moeq.MODE_PREFILL, st)

    with torch.cuda.stream(st):
        for i in range(warmup):
            step(i)
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    n0 = moeq.moeq_launch_count()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for i in range(steps):
                step(i)
    launches = moeq.moeq_launch_count() - n0
    with torch.cuda.stream(st):
        g.replay()
    st.synchronize()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    ms, clk = timed_replays(lambda: g.replay(), 1, st, world, local)
    ms /= steps
    # the same graph replayed for at least min_ms (a long clock record)
    reps = max(1, math.ceil(min_ms / max(ms * steps, 1e-3)))
    ms_long, clk_long = timed_replays(lambda: g.replay(), reps, st, world, local)
    sus_peak, sus_kind = sustained_bf16_peak()
    sustained = {"steps": reps * steps, "timed_ms": ms_long, "ms_per_step": ms_long / (reps * steps),
                 "value": M * world / (ms_long / (reps * steps) / 1e3), "clocks": clk_long.summary(),
                 "layer_tflops": layer_flop_of(workload) / (ms_long / (reps * steps) / 1e3) / 1e12,
                 "peak_tflops": sus_peak, "peak_kind": sus_kind}
    sustained["layer_frac"] = sustained["layer_tflops"] / sus_peak
    # gate/up gather-QMM per launch
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for e in starts + stops:
        e.record(st)
    st.synchronize()
    kg = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(kg, stream=st):
            for i in range(steps):
                moeq.moeq_set_profile_events(starts[i], stops[i])
                step(i)
        moeq.moeq_set_profile_events(None, None)
        kg.replay()
    st.synchronize()
    k_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(starts, stops)) / steps, world)
    n_pairs = M * cfg.K
    gu_flop = 2.0 * n_pairs * 2 * cfg.I * cfg.H
    layer_flop = M * cfg.flops_per_token()
    _, peak_bf16, peak_kind = measured_peaks()
    out = {"workload": workload, "tokens_per_step": M, "steps": steps,
           "value": M * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
           "layer_tflops": layer_flop / (ms / 1e3) / 1e12,
           "layer_frac": layer_flop / (ms / 1e3) / 1e12 / peak_bf16,
           "sustained": sustained,
           "roofline": {"bound": "tensor", "kernel": "k_gqmm gate/up+SwiGLU (fp16 operands)",
                        "achieved": gu_flop / (k_ms / 1e3) / 1e12, "peak": peak_bf16,
                        "unit": "TFLOP/s", "frac": gu_flop / (k_ms / 1e3) / 1e12 / peak_bf16,
                        "traffic": TRAFFIC.get(workload), "flop_per_launch": gu_flop,
                        "ms_per_launch": k_ms,
                        "peak_kind": peak_kind + " bf16 dense (fp16 equal rate)"},
           "gpu_launches": int(launches), "clocks": clk.summary()}
    if want_e2e:
        xh = xs[0].cpu().pin_memory()
        yh = torch.empty((M, cfg.H), dtype=torch.float32).pin_memory()
        xdev = torch.empty((M, cfg.H), dtype=torch.bfloat16, device="cuda")
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            a0.record(st)
            for i in range(steps):
                xdev.copy_(xh, non_blocking=True)
                moeq.moeq_layer_forward(L.desc, xdev, M, y, None, idx, w, ws.buf, ws.bytes,
                                        moeq.MODE_PREFILL, st)
                yh.copy_(y, non_blocking=True)
            a1.record(st)
        st.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(a0.elapsed_time(a1), world) / steps
        out["e2e"] = {"value": M * world / (e2e_ms / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": M * cfg.H * 2, "d2h_bytes_per_step": M * cfg.H * 4}
    out["device_status"] = moeq.moeq_device_status(st)
    g.reset()
    kg.reset()
    del L, ws
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    from quantized_mixture_experts_affine_b200 import moeq, synth
    from quantized_mixture_experts_affine_b200.layer import Workspace, synthetic_layer

    rank, world, local = dist_setup(args.gpus)
    cfg_name, M = WORKLOADS[args.workload]
    cfg = shape(cfg_name)
    if args.workload.startswith("prefill"):
        return run_prefill_main(args, rank, world)
    K, W = args.steps, args.warmup
    assert W >= 3, "at least 3 warm-up steps"
    copies = max(1, args.copies)
    seed = 1000 * rank
    layers = [synthetic_layer(cfg, seed, c) for c in range(copies)]
    total_steps = W + K
    # a fresh token batch per step
    xs = synth.normal_bf16_dev(seed, synth.tag(synth.X, 777), total_steps * M * cfg.H).view(
        total_steps, M, cfg.H)
    ys = torch.empty((copies, M, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((copies, M, cfg.K), dtype=torch.int32, device="cuda")
    wts = torch.empty((copies, M, cfg.K), dtype=torch.float32, device="cuda")
    ws = Workspace(layers[0], M, moeq.MODE_DECODE)
    st = torch.cuda.Stream()
    torch.cuda.synchronize()

    def step(i, stream):
        c = i % copies
        moeq.moeq_layer_forward(layers[c].desc, xs[i], M, ys[c], None, idx[c], wts[c], ws.buf,
                                ws.bytes, moeq.MODE_DECODE, stream)

    # warm-up (also first-call set-up of the library) outside any capture
    with torch.cuda.stream(st):
        for i in range(W):
            step(i, st)
    st.synchronize()

    # capture the K timed steps as CUDA graphs of `copies` steps each
    graphs = []
    n0 = moeq.moeq_launch_count()
    with torch.cuda.stream(st):
        for g0 in range(W, total_steps, copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                for i in range(g0, min(g0 + copies, total_steps)):
                    step(i, st)
            graphs.append(g)
    launches_per_timed_region = moeq.moeq_launch_count() - n0
    # one untimed replay of the first graph (graph upload)
    with torch.cuda.stream(st):
        graphs[0].replay()
    st.synchronize()

    peak_hbm, peak_bf16, peak_kind = measured_peaks()

    def replay_all():
        for g in graphs:
            g.replay()

    # the timed region: exactly the K steps
    ms_total, clk = timed_replays(replay_all, 1, st, world, local)
    ms_step = ms_total / K
    value = M * K * world / (ms_total / 1e3)
    # the same K steps replayed for at least 100 ms (a long clock record)
    reps = max(1, math.ceil(100.0 / max(ms_total, 1e-3)))
    ms_long, clk_long = timed_replays(replay_all, reps, st, world, local)
    sustained = {"steps": reps * K, "timed_ms": ms_long, "ms_per_step": ms_long / (reps * K),
                 "value": M * reps * K * world / (ms_long / 1e3), "clocks": clk_long.summary()}
    # without a graph: the K steps as eager calls through the C ABI, repeated
    # for at least 100 ms (host launch cost included)
    def eager_all():
        for i in range(W, total_steps):
            step(i, st)
    ms_eager1, _ = timed_replays(eager_all, 1, st, world, local)
    reps_e = max(1, math.ceil(100.0 / max(ms_eager1, 1e-3)))
    ms_eager, clk_eager = timed_replays(eager_all, reps_e, st, world, local)
    no_graph = {"steps": reps_e * K, "timed_ms": ms_eager,
                "ms_per_step": ms_eager / (reps_e * K),
                "value": M * reps_e * K * world / (ms_eager / 1e3), "clocks": clk_eager.summary()}

    # routing actually taken in the last steps -> distinct expert bytes per step
    exp_bytes = cfg.expert_bytes()
    gu_bytes_expert = 2 * synth.packed_bytes(cfg.I, cfg.H, cfg.expert_bits, cfg.G)
    sh_gu = 2 * synth.packed_bytes(cfg.shared_I, cfg.H, cfg.shared_bits, cfg.G) if cfg.shared else 0
    idx_np = idx.cpu().numpy()
    distinct = [len(set(idx_np[c].ravel().tolist())) for c in range(copies)]
    mean_distinct = sum(distinct) / len(distinct)
    layer_bytes = cfg.router_bytes() + mean_distinct * exp_bytes + cfg.shared_bytes()
    gu_bytes = mean_distinct * gu_bytes_expert + sh_gu

    # dominant kernel (the gate/up launch): per-launch durations over the same steps,
    # events recorded around it inside captured graphs
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for e in starts + stops:       # create the CUDA events before capture
        e.record(st)
    st.synchronize()
    kgraphs = []
    with torch.cuda.stream(st):
        for g0 in range(W, total_steps, copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                for i in range(g0, min(g0 + copies, total_steps)):
                    moeq.moeq_set_profile_events(starts[i - W], stops[i - W])
                    step(i, st)
            moeq.moeq_set_profile_events(None, None)
            kgraphs.append(g)
        for g in kgraphs:
            g.replay()
    st.synchronize()
    k_ms = sum(a.elapsed_time(b) for a, b in zip(starts, stops)) / K
    k_ms = max_over_ranks(k_ms, world)
    achieved = gu_bytes / (k_ms / 1e3) / 1e9

    # end to end through the public API: pinned host x -> device, forward,
    # y -> pinned host, every step
    e2e = None
    if not args.no_e2e:
        x_host = xs[:K].cpu().pin_memory()
        y_host = torch.empty((K, M, cfg.H), dtype=torch.float32).pin_memory()
        xdev = torch.empty((M, cfg.H), dtype=torch.bfloat16, device="cuda")
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(st):
            e0.record(st)
            for i in range(K):
                c = i % copies
                xdev.copy_(x_host[i], non_blocking=True)
                moeq.moeq_layer_forward(layers[c].desc, xdev, M, ys[c], None, idx[c], wts[c],
                                        ws.buf, ws.bytes, moeq.MODE_DECODE, st)
                y_host[i].copy_(ys[c], non_blocking=True)
            e1.record(st)
        st.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": M * K * world / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": M * cfg.H * 2, "d2h_bytes_per_step": M * cfg.H * 4}
    status = moeq.moeq_device_status(st)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_of(args.workload, world, copies),
        "cuda_graph": True,
        "sustained": sustained,
        "no_graph": no_graph,
        "layer_hbm": {"bytes_per_step": layer_bytes, "achieved_gbs": layer_bytes / (ms_step / 1e3) / 1e9,
                      "peak_gbs": peak_hbm, "frac": layer_bytes / (ms_step / 1e3) / 1e9 / peak_hbm,
                      "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "kernel": gateup_kernel(cfg, M), "achieved": achieved,
                     "peak": peak_hbm, "unit": "GB/s", "frac": achieved / peak_hbm,
                     "traffic": TRAFFIC.get(args.workload), "bytes_per_launch": gu_bytes,
                     "ms_per_launch": k_ms,
                     "peak_kind": peak_kind},
        "e2e": e2e,
        "gpu_launches": int(launches_per_timed_region),
        "clocks": clk.summary(),
        "device_status": status,
    }
    if rank == 0 and not args.no_cpu_baseline:
        smp = OracleSample(cfg, args.cpu_sample)
        dt = smp.run(list(range(args.cpu_sample)))
        line["cpu_baseline"] = {"value": args.cpu_sample / dt, "unit": "tokens/s",
                                "cores": smp.cores(args.cpu_sample), "kind": "oracle",
                                "sample": f"{args.cpu_sample} tokens of {args.workload}, "
                                          f"one oracle call ({dt:.2f} s)"}
    for g in graphs + kgraphs:
        g.reset()
    if not args.no_prefill:
        del layers
        torch.cuda.empty_cache()
        line["prefill"] = measure_prefill(args.prefill_workload, max(3, min(K, 20)), W, world,
                                          seed, want_e2e=not args.no_e2e)
        line["prefill"]["config"] = config_of(args.prefill_workload, world, copies)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_prefill_main(args, rank, world):
    """A prefill workload as the main line: value = tokens/s of one-shot calls."""
    cfg_name, M = WORKLOADS[args.workload]
    assert args.warmup >= 3, "at least 3 warm-up steps"
    p = measure_prefill(args.workload, args.steps, args.warmup, world, 1000 * rank,
                        want_e2e=not args.no_e2e)
    line = {"metric": METRIC, "value": p["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": p["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": config_of(args.workload, world, args.copies), "cuda_graph": True,
            "layer_tflops": p["layer_tflops"], "layer_frac": p["layer_frac"],
            "sustained": p["sustained"], "roofline": p["roofline"], "e2e": p.get("e2e"),
            "gpu_launches": p["gpu_launches"], "clocks": p["clocks"],
            "device_status": p["device_status"]}
    if rank == 0 and not args.no_cpu_baseline:
        smp = OracleSample(shape(cfg_name), args.cpu_sample)
        dt = smp.run(list(range(args.cpu_sample)))
        line["cpu_baseline"] = {"value": args.cpu_sample / dt, "unit": "tokens/s",
                                "cores": smp.cores(args.cpu_sample), "kind": "oracle",
                                "sample": f"{args.cpu_sample} tokens of {args.workload}, "
                                          f"one oracle call ({dt:.2f} s)"}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ per-config table
# (row, shape, tokens per call, kind): kind "layer" = moeq_layer_forward in
# AUTO mode; "zipf" = moeq_route_topk on router logits drawn with a Zipf
# (s = 1.1) expert load, then moeq_expert_ffn in AUTO mode; "qmv" = the
# standalone 8-bit router qmv 2816 -> 128.
SWEEP = [
    ("C1", "tiny", 1, "layer"), ("C1", "tiny", 3, "layer"), ("C1", "tiny", 5, "layer"),
    ("C2", "decode_30b", 1, "layer"), ("C2", "router_2816", 1, "qmv"),
    ("C3", "decode_397b", 1, "layer"), ("C3", "decode_397b", 8, "layer"),
    ("C3", "decode_397b", 64, "layer"),
    ("C4", "prefill_8bit", 16032, "layer"), ("C4", "prefill_8bit", 16068, "layer"),
    ("C4", "prefill_8bit", 16384, "layer"),
    ("C5", "mixed_2bit", 1, "zipf"), ("C5", "mixed_2bit", 256, "zipf"),
    ("C5", "mixed_2bit", 4096, "zipf"),
]


def sweep_row(row, name, M, kind, copies, seed=0):
    """GPU time per call (graph replays, >= 100 ms), tokens/s, roofline
    fraction, and the oracle on a token sample (1 core and all cores)."""
    import numpy as np
    import torch
    from quantized_mixture_experts_affine_b200 import moeq, synth
    from quantized_mixture_experts_affine_b200.layer import Workspace, synthetic_layer
    peak_hbm, peak_bf16, peak_kind = measured_peaks()
    st = torch.cuda.Stream()
    out = {"row": row, "shape": name, "tokens_per_call": M, "kind": kind}
    if kind == "qmv":
        H, E = 2816, 128
        Ts = [synth.tensor_dev(seed, synth.tag(synth.ROUTER, 50 + c), 1, E, H, 8, 64)
              for c in range(copies)]
        descs = [moeq.qtensor(t.w, t.s, t.b, E, H, 8, 64, 1) for t in Ts]
        x = synth.normal_bf16_dev(seed, synth.tag(synth.X, 51), H).view(1, H)
        y = torch.empty((1, E), device="cuda")
        call = lambda i: moeq.moeq_qmv(descs[i % copies], 0, x, 1, y, st)
        nbytes = E * H + 4 * E * (H // 64)
    else:
        cfg = shape(name)
        layers = [synthetic_layer(cfg, seed, c) for c in range(copies)]
        xs = synth.normal_bf16_dev(seed, synth.tag(synth.X, 52), copies * M * cfg.H).view(
            copies, M, cfg.H)
        y = torch.empty((M, cfg.H), device="cuda")
        idx = torch.empty((M, cfg.K), dtype=torch.int32, device="cuda")
        w = torch.empty((M, cfg.K), device="cuda")
        ws = Workspace(layers[0], M, moeq.MODE_AUTO)
        if kind == "zipf":
            lg, _ = synth.zipf_logits_host(seed, synth.tag(synth.LOGITS, 53), M, cfg.E, 1.1)
            logits = torch.from_numpy(np.ascontiguousarray(lg)).cuda()

            def call(i):
                moeq.moeq_route_topk(logits, M, cfg.E, cfg.K, cfg.renorm, cfg.router_scale, idx,
                                     w, st)
                moeq.moeq_expert_ffn(layers[i % copies].desc, xs[i % copies], M, idx, w, None, y,
                                     ws.buf, ws.bytes, moeq.MODE_AUTO, st)
        else:
            def call(i):
                moeq.moeq_layer_forward(layers[i % copies].desc, xs[i % copies], M, y, None, idx,
                                        w, ws.buf, ws.bytes, moeq.MODE_AUTO, st)
    # the inputs are drawn on the current stream: done before st uses them
    torch.cuda.synchronize()
    with torch.cuda.stream(st):
        for i in range(3):
            call(i)
    st.synchronize()
    n = copies if M < 1024 else 2
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for i in range(n):
                call(i)
        g.replay()
    st.synchronize()
    ms1, _ = timed_replays(lambda: g.replay(), 1, st, 1, 0)
    reps = max(1, math.ceil(100.0 / max(ms1, 1e-3)))
    ms, clk = timed_replays(lambda: g.replay(), reps, st, 1, 0)
    ms_call = ms / (reps * n)
    out.update({"gpu_ms": ms_call, "tokens_per_s": M / (ms_call / 1e3), "timed_ms": ms,
                "clocks": clk.summary(), "device_status": moeq.moeq_device_status(st)})
    if kind == "qmv":
        out["roofline"] = {"bound": "hbm", "bytes": nbytes,
                           "frac": nbytes / (ms_call / 1e3) / 1e9 / peak_hbm}
    else:
        # both rooflines: the weight bytes the call must stream (router
        # unless the routing is given, the distinct routed experts, the
        # shared expert) and the layer's FLOPs; the bound is the larger
        distinct = len(set(idx.cpu().numpy().ravel().tolist()))
        nbytes = (0 if kind == "zipf" else cfg.router_bytes()) + distinct * cfg.expert_bytes() \
            + cfg.shared_bytes()
        flop = M * cfg.flops_per_token() - (2 * M * cfg.E * cfg.H if kind == "zipf" else 0)
        hbm = nbytes / (ms_call / 1e3) / 1e9 / peak_hbm
        ten = flop / (ms_call / 1e3) / 1e12 / peak_bf16
        out["roofline"] = {"bound": "hbm" if hbm >= ten else "tensor", "bytes": nbytes,
                           "distinct_experts": distinct, "flop": flop, "hbm_frac": hbm,
                           "tensor_frac": ten, "frac": max(hbm, ten)}
    out["path"] = ("decode" if kind != "qmv" and M <= 64 and M * cfg.K <= 96 else
                   "prefill" if kind != "qmv" else "qmv")
    out["roofline"]["peak_kind"] = peak_kind
    del g
    torch.cuda.empty_cache()
    if kind != "qmv":
        smp = OracleSample(cfg, 16)
        t1 = smp.run([0], threads=1)
        tn = smp.run(list(range(16)))
        out["oracle"] = {"one_core_tokens_per_s": 1 / t1, "all_cores_tokens_per_s": 16 / tn,
                         "cores": smp.cores(16), "sample": "1 token (1 core), 16 tokens (all cores)"}
    return out


def run_sweep(args):
    import platform
    import torch
    torch.cuda.set_device(0)
    head = {"sweep": "per-config table", "gpu": torch.cuda.get_device_name(0),
            "host_cores": os.cpu_count(), "cpu": platform.processor() or platform.machine()}
    print(json.dumps(head), flush=True)
    for row, name, M, kind in SWEEP:
        if args.sweep_rows and row not in args.sweep_rows.split(","):
            continue
        print(json.dumps(sweep_row(row, name, M, kind, args.copies)), flush=True)


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
