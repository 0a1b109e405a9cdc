"""Benchmark of the routed int4 expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config dsv2lite] [--tokens 8]

One step = one forward of the whole layer (router, top-k, bucketing, gate/up +
SwiGLU, down projection, weighted combine) over one batch of synthetic tokens,
inputs already resident in HBM.  The default workload is the
DeepSeek-V2-Lite-shaped decode layer (hidden 2048, inter 1408, 64 routed
experts top-6 + 2 shared, 64 slots bound in a random permutation) at 8 tokens,
a fresh seeded batch each step.  L2 is flushed between steps (a 256 MiB write,
then a 256 MiB read so the written lines leave L2 before the step), outside the
per-step CUDA-event brackets.  N > 1 runs N independent
replicas (the layer has no cross-GPU step on one GPU's worth of experts), one
process per GPU; value = all ranks' tokens / the slowest rank's time.

Printed (rank 0): one JSON line with metric, value, unit, roofline of the
dominant kernel (gate/up + SwiGLU, HBM-bound), e2e (host buffers through the
C interface, copies inside the timed region), cpu_baseline (the CPU oracle on
a bounded sample), clocks sampled during the timed region, gpu_launches.

--impl reference times the CPU oracle on this host on the same workload (one
bounded sample per step) and prints the same JSON line with "impl":
"reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from quantized_routed_expert_04_b200 import synth  # noqa: E402

METRIC = "MoE-layer tokens/s"
SMALL_T = 64  # the library's decode kernels serve up to this many tokens
UNIT = "tokens/s"
PHASES = ("router", "topk", "bucket", "pack", "gate_up", "down", "combine", "gather")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="dsv2lite", choices=sorted(synth.CONFIGS))
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args()
    if a.tokens is None:
        a.tokens = {"dsv2lite": 8}.get(a.config, synth.CONFIGS[a.config].tokens[-1])
    a.warmup = max(3, a.warmup)
    return a


def workload_desc(cfg, T):
    return {"workload": "%s, %d tokens" % (cfg.description, T), "hidden": cfg.hidden,
            "inter": cfg.inter, "n_experts": cfg.n_experts, "top_k": cfg.top_k,
            "n_shared": cfg.n_shared, "n_slots": cfg.n_slots, "tokens": T,
            "routing": cfg.routing if cfg.routing == "softmax" else
            "%s (correction bias, routed scale %g)" % (cfg.routing, cfg.routed_scale)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica_seed(seed, rank):
    """Each replica draws its own token stream (the weights are shared)."""
    return seed + rank


def max_over_ranks(value, world, device):
    """The slowest rank's time: every rank calls this in the same order."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank, world, ms_slowest):
    """Replicas: every rank processes its own batch; all tokens / slowest time."""
    return tokens_per_rank * world / (ms_slowest / 1000.0)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """NVML samples of the SM clock and throttle reasons on one GPU."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, index, period=0.01):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period, self.index = period, index
        self.stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = fn(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------- oracle leg
def oracle_step_time(cfg, blobs, W, b, x_bits, corr=None):
    import oracle
    E, S = cfg.n_experts, cfg.n_shared
    t0 = time.perf_counter()
    if cfg.routing == "sigmoid":
        _, idx, w = oracle.route_sigmoid(x_bits, W, b, corr, cfg.routed_scale, cfg.top_k)
    else:
        _, idx, w = oracle.route(x_bits, W, b, cfg.top_k)
    st, _ = oracle.forward_routed(x_bits, cfg.hidden, cfg.inter, E, cfg.top_k, np.arange(E),
                                  [blobs[e] for e in range(E)], [blobs[E + i] for i in range(S)],
                                  idx, w)
    assert st == oracle.OK
    return time.perf_counter() - t0


def cpu_sample_tokens(cfg, T):
    """Tokens per oracle sample: all of a decode batch; a strided subset of a
    prefill batch (the per-token work is independent)."""
    return T if T <= 16 else 8


def run_cpu_baseline(cfg, blobs, W, b, T, seed, budget_s=20.0, max_steps=8, corr=None):
    n = cpu_sample_tokens(cfg, T)
    total, toks, steps = 0.0, 0, 0
    while steps < max_steps and (total < budget_s or steps == 0):
        x = synth.make_x(cfg, T, seed, step=10_000 + steps)
        if n < T:
            x = x[np.linspace(0, T - 1, n).astype(int)]
        total += oracle_step_time(cfg, blobs, W, b, x, corr)
        toks += n
        steps += 1
        if total / steps * (steps + 1) > budget_s * 1.5:
            break
    sample = ("%d oracle step(s) of %d token(s)" % (steps, n) +
              ("" if n == T else " (strided subset of a %d-token batch)" % T))
    return {"value": toks / total, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
            "seconds": round(total, 3)}


def reference_arm(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cfg = synth.CONFIGS[args.config]
    T = args.tokens
    blobs = synth.make_all_blobs(cfg, args.seed)
    W, b = synth.make_router(cfg, args.seed)
    corr = synth.make_correction_bias(cfg, args.seed) if cfg.routing == "sigmoid" else None
    n = cpu_sample_tokens(cfg, T)
    per_step_budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup if args.warmup < 3 else 1):
        x = synth.make_x(cfg, T, args.seed, step=20_000 + i)[:n]
        oracle_step_time(cfg, blobs, W, b, x, corr)
    times = []
    t_start = time.perf_counter()
    for s in range(args.steps):
        x = synth.make_x(cfg, T, args.seed, step=s)
        if n < T:
            x = x[np.linspace(0, T - 1, n).astype(int)]
        times.append(oracle_step_time(cfg, blobs, W, b, x, corr))
        if time.perf_counter() - t_start > per_step_budget * args.steps:
            break
    k = len(times)
    tok_s = n * k / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": 1,
            "steps": k, "warmup": args.warmup, "ms_per_step": 1000 * sum(times) / k,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded)", "config": workload_desc(cfg, T),
            "cpu_baseline": {"value": tok_s, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": "%d step(s) of %d token(s)%s" % (
                                 k, n, "" if n == T else " (strided subset)")},
            "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ----------------------------------------------------------------- our arm
def traffic_from_profile(kernel_files, key):
    """dram bytes per launch recorded in profiles/<key>.md, if the kernel
    sources still hash to the recorded value."""
    path = os.path.join(ROOT, "profiles", key + ".md")
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for f in kernel_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()[:16]
    rec = {}
    for line in open(path):
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            rec[k.strip()] = v.strip().strip("`")
    if rec.get("source_sha256_16") != digest:
        return None
    try:
        return float(rec["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    import torch
    import torch.distributed as dist

    from quantized_routed_expert_04_b200 import binding, build
    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    build.build()
    binding.load_library()
    cfg = synth.CONFIGS[args.config]
    T = args.tokens
    E, S = cfg.n_experts, cfg.n_shared
    seed = replica_seed(args.seed, rank)

    # --- the layer: every blob resident (slots bound in a seeded permutation),
    # or, for a layer with fewer slots than experts, an LRU arena filled per
    # step from a pinned host pool of all experts (copies on a side stream,
    # timed apart from the layer)
    blobs = synth.make_all_blobs(cfg, args.seed)
    W, b = synth.make_router(cfg, args.seed)
    W_dev = torch.from_numpy(W).cuda()
    b_dev = None if b is None else torch.from_numpy(b).cuda()
    paged = cfg.n_slots < E
    layer = binding.StrataMoE(cfg.hidden, cfg.inter, E, cfg.top_k, S, cfg.n_slots)
    layer.set_router(W_dev, b_dev)
    corr = None
    if cfg.routing == "sigmoid":
        corr = synth.make_correction_bias(cfg, args.seed)
        corr_dev = torch.from_numpy(corr).cuda()
        layer.set_routing(binding.ROUTE_SIGMOID, corr_dev, cfg.routed_scale)
    B_e = synth.expert_bytes(cfg.hidden, cfg.inter)
    if paged:
        dev_shared = torch.from_numpy(blobs[E:]).cuda()
        for i in range(S):
            layer.bind_shared(i, dev_shared[i])
        pool = torch.from_numpy(np.ascontiguousarray(blobs[:E]).reshape(-1)).pin_memory()
        arena_mem = torch.empty(cfg.n_slots * B_e, dtype=torch.uint8, device="cuda")
        arena = binding.Arena(layer, pool, arena_mem)
        copy_stream = torch.cuda.Stream()
    else:
        dev_blobs = torch.from_numpy(blobs).cuda()
        for i in range(S):
            layer.bind_shared(i, dev_blobs[E + i])
        for s, e in enumerate(synth.make_slot_permutation(cfg, args.seed)):
            layer.bind_slot(s, int(e), dev_blobs[int(e)])
    layer.reserve(T)

    steps_total = args.warmup + args.steps
    n_batches = min(steps_total, 64)
    xs = [torch.from_numpy(synth.make_x(cfg, T, seed, step=s).view(np.int16)).cuda()
          .view(torch.bfloat16) for s in range(n_batches)]
    out = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")

    # distinct experts per batch (for the algorithmic byte count), via route()
    idx_t = torch.empty(T, cfg.top_k, dtype=torch.int32, device="cuda")
    w_t = torch.empty(T, cfg.top_k, dtype=torch.float32, device="cuda")
    distinct = []
    for x in xs:
        layer.route(x, None, idx_t, w_t)
        distinct.append(len(set(idx_t.cpu().numpy().reshape(-1).tolist())))
    gateup_bytes = [(d + S) * 2 * cfg.inter * cfg.hidden * 9 // 16 for d in distinct]
    step_bytes = [(d + S) * B_e for d in distinct]
    flops_per_step = 6 * cfg.hidden * cfg.inter * T * (cfg.top_k + S)

    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    clean = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    sink = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def flush_l2(i):
        # write a buffer larger than L2, then read another one so that the
        # flush's dirty lines are written back here, outside the timed region
        flush.fill_(float(i))
        torch.sum(clean, dim=0, out=sink.view(()))

    idx_host = torch.empty(T, cfg.top_k, dtype=torch.int32).pin_memory()
    paging = {"hits": 0, "misses": 0, "bytes": 0, "copy_ms": 0.0, "steps": 0}

    def step(i, inner=None, x=None):
        """One forward.  Paged: route, read the ids, make them resident,
        forward with the routing; `inner` (4 events) brackets the two kernel
        phases so that the copies in between are timed apart."""
        x = xs[i % n_batches] if x is None else x
        if not paged:
            layer.forward(x, out)
            return
        if inner:
            inner[0].record(stream)
        layer.route(x, None, idx_t, w_t)
        if inner:
            inner[1].record(stream)
        idx_host.copy_(idx_t)
        hits, misses, nbytes = arena.ensure(idx_host.numpy().reshape(-1), stream=stream,
                                            copy_stream=copy_stream)
        if inner:
            inner[2].record(stream)
        layer.forward_routed(x, idx_t, w_t, out)
        if inner:
            inner[3].record(stream)
            paging["hits"] += hits
            paging["misses"] += misses
            paging["bytes"] += nbytes
            paging["copy_ms"] += arena.copy_ms()
            paging["steps"] += 1

    for i in range(args.warmup):
        flush_l2(i)
        step(i)
    torch.cuda.synchronize()
    st, bits = layer.status()
    if int(st) != 0:
        raise RuntimeError("device status %s bits %d" % (st, bits))

    # --- timed region: the forward exactly as a user runs it (consecutive
    # kernels overlap through programmatic dependent launch); step events on
    # the launch stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    inner = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush_l2(i)
            ev[i][0].record(stream)
            step(args.warmup + i, inner[i] if paged else None)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    # --- kernel pass: the same steps again with an event pair around every
    # kernel (which serialises the launches), for per-kernel times and the
    # dominant kernel's roofline
    kp_steps = min(args.steps, 50)
    binding.strata_moe_profile(layer.h, True)
    binding.strata_moe_profile_read(layer.h)
    for i in range(kp_steps):
        flush_l2(i)
        step(args.warmup + i)
    torch.cuda.synchronize()
    prof = binding.strata_moe_profile_read(layer.h)
    binding.strata_moe_profile(layer.h, False)
    if paged:  # layer kernels only: routing + forward, not the copies between them
        step_ms = [e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in inner]
    else:
        step_ms = [a.elapsed_time(bb) for a, bb in ev]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world, "cuda")
    value = whole_job_tokens_per_s(T, world, ms)

    # --- dominant kernel roofline (gate/up + SwiGLU): the HBM-bound decode
    # kernel for small batches, the tensor-core kernel for large ones
    peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(peaks_path):
        peaks = json.load(open(peaks_path))
        hbm_peak, tc_peak, peak_src = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"]), \
            "measured"
    else:
        hbm_peak, tc_peak, peak_src = 6650.0, 1590.0, "fallback"
    n_gu, ms_gu = prof["gate_up"]
    timed_ids = [(args.warmup + i) % n_batches for i in range(args.steps)]
    kp_ids = timed_ids[:kp_steps]
    avg_gu_ms = ms_gu / max(1, n_gu)
    alg_step = sum(step_bytes[j] for j in timed_ids) / len(timed_ids)
    if T <= SMALL_T:
        alg_gu = sum(gateup_bytes[j] for j in kp_ids) / len(kp_ids)
        traffic = traffic_from_profile(
            ["quantized_routed_expert_04_b200/csrc/expert_mma.cu",
             "quantized_routed_expert_04_b200/csrc/common.cuh"],
            "expert_mma_gateup_%s_t%d" % (args.config, T))
        roofline = {"kernel": "expert_mma_kernel<gate/up+SwiGLU>", "bound": "hbm",
                    "achieved": alg_gu / (avg_gu_ms / 1000.0) / 1e9, "peak": hbm_peak,
                    "unit": "GB/s", "peak_source": peak_src + " (copy kernel)",
                    "algorithmic_bytes_per_launch": alg_gu}
    else:
        alg_gu = 4.0 * cfg.hidden * cfg.inter * T * (cfg.top_k + S)
        traffic = traffic_from_profile(
            ["quantized_routed_expert_04_b200/csrc/prefill_tc.cu",
             "quantized_routed_expert_04_b200/csrc/common.cuh"],
            "expert_tc_gateup_%s_t%d" % (args.config, T))
        roofline = {"kernel": "expert_tc_kernel<gate/up+SwiGLU>", "bound": "tensor",
                    "achieved": alg_gu / (avg_gu_ms / 1000.0) / 1e12, "peak": tc_peak,
                    "unit": "TFLOP/s", "peak_source": peak_src + " (dense bf16 GEMM burst; "
                    "f16 has the same rate)", "algorithmic_flops_per_launch": alg_gu}
    roofline["frac"] = roofline["achieved"] / roofline["peak"]
    roofline["traffic"] = traffic
    roofline["avg_launch_ms"] = avg_gu_ms
    roofline["timing"] = ("CUDA events around every launch, in a pass of %d of the timed steps "
                          "run again right after the timed region (launches serialised)" % kp_steps)
    phase_ms = {k: round(v[1] / max(1, v[0]), 5) for k, v in prof.items() if v[0]}
    launches = sum(v[0] for v in prof.values()) * args.steps // kp_steps  # per step x K

    # --- end to end through the C interface with host buffers
    x_host = [torch.empty(T, cfg.hidden, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    for j, xh in enumerate(x_host):
        xh.copy_(xs[j % n_batches].cpu())
    out_host = torch.empty(T, cfg.hidden, dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty_like(xs[0])
    e2e_steps = max(10, min(args.steps, 200))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        flush_l2(i)
        e2e_ev[i][0].record(stream)
        x_stage.copy_(x_host[i % 4], non_blocking=True)
        step(i, x=x_stage)   # paged: includes the host routing read and the copies
        out_host.copy_(out, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(bb) for a, bb in e2e_ev) / e2e_steps, world,
                            "cuda")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(cfg, blobs, W, b, T, args.seed, corr=corr)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4 weights x f16 activations, f32 accumulate (router f64)",
            "data": "synthetic (seeded, resident in HBM)",
            "config": dict(workload_desc(cfg, T),
                           l2="flushed between steps: 256 MiB write, then 256 MiB read (outside "
                              "the per-step event brackets)",
                           parallelism="replicas" if world > 1 else "1 GPU"),
            "expert_weight_gbs": alg_step / (ms / 1000.0) / 1e9,
            "expert_weight_frac_of_hbm": alg_step / (ms / 1000.0) / 1e9 / hbm_peak,
            "tflops": flops_per_step / (ms / 1000.0) / 1e12,
            "roofline": roofline,
            "expert_gemm_tflops": (6.0 * cfg.hidden * cfg.inter * T * (cfg.top_k + S) /
                                   ((prof["gate_up"][1] + prof["down"][1]) /
                                    max(1, prof["gate_up"][0]) / 1000.0) / 1e12),
            "phase_ms_per_launch": phase_ms,
            "e2e": {"value": whole_job_tokens_per_s(T, world, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": T * cfg.hidden * 2,
                    "d2h_bytes_per_step": T * cfg.hidden * 2, "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
            "wall_s_timed_region": t_wall,
        }
        if paged:
            n = max(1, paging["steps"])
            line["paging"] = {
                "n_slots": cfg.n_slots, "note": "layer time (value) excludes the expert copies; "
                "e2e includes them and the host read of the routing",
                "hits_per_step": paging["hits"] / n, "misses_per_step": paging["misses"] / n,
                "copy_bytes_per_step": paging["bytes"] / n,
                "copy_ms_per_step": paging["copy_ms"] / n,
                "copy_gbs": (paging["bytes"] / max(paging["copy_ms"], 1e-9) / 1e6)}
            line["data"] = "synthetic (seeded); %d of %d experts resident, the rest in pinned " \
                           "host memory" % (cfg.n_slots, E)
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line))
    layer.close()
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
