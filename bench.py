"""Benchmark of the routed int4 expert layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config prefill] [--tokens 8192] [--no-subrecords]

One step = one forward of the whole layer (router, top-k, bucketing, gate/up +
SwiGLU, down projection, weighted combine) over one batch of synthetic tokens,
inputs already resident in HBM.

The headline workload (the largest single-GPU layer configuration) is the
prefill layer: hidden 4096, inter 2048, 256 routed experts top-8 + 1 shared,
8192 tokens with a Zipf(0.8) router bias, every expert resident.  Its line
carries the layer's tokens/s (value), the grouped GEMMs' TFLOP/s against the
dense tensor-core peak (roofline), end-to-end tokens/s with host buffers
(e2e), the CPU oracle on a bounded sample (cpu_baseline) and the SM clocks
sampled under load.  The same line carries one sub-record per decode
workload -- DeepSeek-V2-Lite-shaped (1 and 8 tokens), Mixtral-shaped (1, 4,
16 tokens) and the wide 256-expert layer over a 64-slot arena (1 and 4 tokens,
expert copies from pinned host memory timed apart) -- each with its tokens/s,
expert-weight GB/s against the HBM peak, roofline and e2e.

L2 is flushed between steps (a 256 MiB write, then a 256 MiB read so the
written lines leave L2 before the step), outside the per-step CUDA-event
brackets.  A fresh seeded batch of tokens is used per step.  N > 1 runs N
independent replicas (one process per GPU; the layer has no cross-GPU step);
value = all ranks' tokens / the slowest rank's time.

--impl reference times the CPU oracle on this host on the same workload (a
strided sample of tokens per step) and prints the same JSON line with "impl":
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

METRIC = "MoE-layer tokens/s; expert-weight HBM GB/s vs peak; prefill TFLOP/s"
SMALL_T = 64  # the library's decode kernels serve up to this many tokens
UNIT = "tokens/s"
HEADLINE = ("prefill", 8192)
SUBRECORDS = [("dsv2lite", 1), ("dsv2lite", 8), ("mixtral", 1), ("mixtral", 4), ("mixtral", 16),
              ("wide", 1), ("wide", 4)]
L2_NOTE = ("flushed between steps: 256 MiB write, then 256 MiB read (outside the per-step "
           "event brackets)")
NOMINAL_HBM_GBS = 8000.0   # the HBM figure the targets are stated against


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=HEADLINE[0], choices=sorted(synth.CONFIGS))
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-subrecords", action="store_true",
                    help="only the headline workload (profiler runs)")
    ap.add_argument("--sub-steps", type=int, default=1000, help="timed steps per sub-record")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args(argv)
    if a.tokens is None:
        a.tokens = {"dsv2lite": 8}.get(a.config, synth.CONFIGS[a.config].tokens[-1])
    a.warmup = max(3, a.warmup)
    a.subrecords = (not a.no_subrecords) and (a.config, a.tokens) == HEADLINE
    return a


def workload_desc(cfg, T):
    return {"workload": "%s, %d tokens" % (cfg.description, T), "hidden": cfg.hidden,
            "inter": cfg.inter, "n_experts": cfg.n_experts, "top_k": cfg.top_k,
            "n_shared": cfg.n_shared, "n_slots": cfg.n_slots, "tokens": T,
            "routing": cfg.routing if cfg.routing == "softmax" else
            "%s (correction bias, routed scale %g)" % (cfg.routing, cfg.routed_scale)}


def config_desc(cfg, T, world):
    """The `config` object, identical for both arms."""
    return dict(workload_desc(cfg, T), l2=L2_NOTE,
                parallelism="%d independent replicas" % world if world > 1 else "1 GPU")


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


def host_info():
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"host_cpu_model": model, "host_cpu_count": os.cpu_count()}


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """NVML samples of the SM clock and throttle reasons on one GPU, taken
    every 10 ms for the whole run; window() summarises the samples between
    two marks."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, index, period=0.01):
        self.samples, self.ok = [], False   # (sm_mhz, reasons set)
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
        fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = fn(self.h)
                self.samples.append((mhz, {n for b, n in self.REASONS.items() if r & b}))
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

    def mark(self):
        return len(self.samples)

    def window(self, start, end=None):
        s = self.samples[start:end]
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, r in s:
            reasons |= r
        return {"sm_mhz": statistics.median(m for m, _ in s), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(s)}


# ----------------------------------------------------------------- oracle leg
def strided_sample(T, n):
    return np.linspace(0, T - 1, n).astype(int) if n < T else np.arange(T)


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


def run_cpu_baseline(cfg, blobs, W, b, T, seed, budget_s=12.0, corr=None):
    """The oracle (single thread) on a bounded sample of the workload: whole
    decode batches, or strided tokens of a prefill batch sized to about
    budget_s of work (the per-token work is independent)."""
    if T <= 16:
        n, steps, total = T, 0, 0.0
        while steps < 8 and (total < budget_s or steps == 0):
            total += oracle_step_time(cfg, blobs, W, b, synth.make_x(cfg, T, seed, 10_000 + steps),
                                      corr)
            steps += 1
            if total / steps * (steps + 1) > budget_s * 1.5:
                break
        toks, sample = n * steps, "%d oracle step(s) of the %d-token batch" % (steps, T)
    else:
        x = synth.make_x(cfg, T, seed, step=10_000)
        probe = oracle_step_time(cfg, blobs, W, b, x[strided_sample(T, 2)], corr) / 2
        n = int(min(T, max(2, budget_s / max(probe, 1e-6))))
        total = oracle_step_time(cfg, blobs, W, b, x[strided_sample(T, n)], corr)
        toks = n
        sample = "%d strided tokens of a %d-token batch (per-token work is independent)" % (n, T)
    out = {"value": toks / total, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
           "seconds": round(total, 3)}
    out.update(host_info())
    return out


def reference_arm(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    cfg = synth.CONFIGS[args.config]
    T = args.tokens
    blobs = synth.make_all_blobs(cfg, args.seed)
    W, b = synth.make_router(cfg, args.seed)
    corr = synth.make_correction_bias(cfg, args.seed) if cfg.routing == "sigmoid" else None
    n = T if T <= 16 else 2     # tokens per step: a decode batch, or 2 strided prefill tokens
    rows = strided_sample(T, n)
    for i in range(min(args.warmup, 1)):
        oracle_step_time(cfg, blobs, W, b, synth.make_x(cfg, T, args.seed, 20_000 + i)[rows], corr)
    times = []
    budget = max(30.0, 3.0 * args.steps)
    t_start = time.perf_counter()
    for s in range(args.steps):
        times.append(oracle_step_time(cfg, blobs, W, b,
                                      synth.make_x(cfg, T, args.seed, step=s)[rows], corr))
        if time.perf_counter() - t_start > budget:
            break
    k = len(times)
    tok_s = n * k / sum(times)
    sample = "%d step(s) of %s" % (k, "the %d-token batch" % T if n == T else
                                   "%d strided tokens of the %d-token batch" % (n, T))
    cpu = {"value": tok_s, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample}
    cpu.update(host_info())
    line = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": UNIT, "n_gpus": world,
            "steps": k, "warmup": args.warmup, "ms_per_step": 1000 * sum(times) / k,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded)", "config": config_desc(cfg, T, world),
            "cpu_baseline": cpu,
            "e2e": {"value": tok_s, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ----------------------------------------------------------------- our arm
def traffic_from_profile(kernel_files, key):
    """DRAM bytes per launch recorded in profiles/<key>.md, if the kernel
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


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm": float(p["hbm_gbs"]), "tc": float(p["bf16_tflops"]),
                "tc_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm": 6650.0, "tc": 1590.0, "tc_sustained": 1400.0, "source": "fallback"}


KERNEL_SOURCES = {
    "decode": ["quantized_routed_expert_04_b200/csrc/decode_fused.cu",
               "quantized_routed_expert_04_b200/csrc/common.cuh"],
    "prefill": ["quantized_routed_expert_04_b200/csrc/prefill_tc.cu",
                "quantized_routed_expert_04_b200/csrc/common.cuh"],
}


class Workload:
    """One layer configuration on the device: blobs bound (or paged through
    an arena), a stream of seeded token batches and the per-step forward."""

    def __init__(self, cfg, T, seed, rank, n_batches):
        import torch

        from quantized_routed_expert_04_b200 import binding
        self.torch, self.cfg, self.T = torch, cfg, T
        E, S = cfg.n_experts, cfg.n_shared
        self.blobs = synth.make_all_blobs(cfg, seed)
        self.W, self.b = synth.make_router(cfg, seed)
        self.W_dev = torch.from_numpy(self.W).cuda()
        self.b_dev = None if self.b is None else torch.from_numpy(self.b).cuda()
        self.paged = cfg.n_slots < E
        self.layer = binding.StrataMoE(cfg.hidden, cfg.inter, E, cfg.top_k, S, cfg.n_slots)
        self.layer.set_router(self.W_dev, self.b_dev)
        self.corr = None
        if cfg.routing == "sigmoid":
            self.corr = synth.make_correction_bias(cfg, seed)
            self.corr_dev = torch.from_numpy(self.corr).cuda()
            self.layer.set_routing(binding.ROUTE_SIGMOID, self.corr_dev, cfg.routed_scale)
        B_e = synth.expert_bytes(cfg.hidden, cfg.inter)
        if self.paged:
            self.dev_shared = torch.from_numpy(self.blobs[E:]).cuda()
            for i in range(S):
                self.layer.bind_shared(i, self.dev_shared[i])
            self.pool = torch.from_numpy(np.ascontiguousarray(self.blobs[:E]).reshape(-1)).pin_memory()
            self.arena_mem = torch.empty(cfg.n_slots * B_e, dtype=torch.uint8, device="cuda")
            self.arena = binding.Arena(self.layer, self.pool, self.arena_mem)
            self.copy_stream = torch.cuda.Stream()
        else:
            self.dev_blobs = torch.from_numpy(self.blobs).cuda()
            for i in range(S):
                self.layer.bind_shared(i, self.dev_blobs[E + i])
            for s, e in enumerate(synth.make_slot_permutation(cfg, seed)):
                self.layer.bind_slot(s, int(e), self.dev_blobs[int(e)])
        self.layer.reserve(T)
        self.n_batches = n_batches
        self.xs = [torch.from_numpy(synth.make_x(cfg, T, replica_seed(seed, rank), step=s)
                                    .view(np.int16)).cuda().view(torch.bfloat16)
                   for s in range(n_batches)]
        self.out = torch.empty(T, cfg.hidden, dtype=torch.bfloat16, device="cuda")
        self.idx_t = torch.empty(T, cfg.top_k, dtype=torch.int32, device="cuda")
        self.w_t = torch.empty(T, cfg.top_k, dtype=torch.float32, device="cuda")
        self.idx_host = torch.empty(T, cfg.top_k, dtype=torch.int32).pin_memory()
        self.paging = {"hits": 0, "misses": 0, "bytes": 0, "copy_ms": 0.0, "steps": 0}
        # distinct routed experts per batch (the algorithmic byte count of a
        # decode step), from the library's own routing
        self.distinct = []
        if T <= SMALL_T:
            for x in self.xs:
                self.layer.route(x, None, self.idx_t, self.w_t)
                self.distinct.append(len(set(self.idx_t.cpu().numpy().reshape(-1).tolist())))

    def step(self, i, inner=None, x=None, record=False):
        """One forward.  Paged: route, read the ids on the host, make them
        resident, forward with the routing; `inner` (4 events) brackets the
        two kernel phases so that the copies in between are timed apart."""
        stream = self.torch.cuda.current_stream()
        x = self.xs[i % self.n_batches] if x is None else x
        if not self.paged:
            self.layer.forward(x, self.out)
            return
        if inner:
            inner[0].record(stream)
        self.layer.route(x, None, self.idx_t, self.w_t)
        if inner:
            inner[1].record(stream)
        self.idx_host.copy_(self.idx_t)
        hits, misses, nbytes = self.arena.ensure(self.idx_host.numpy().reshape(-1),
                                                 stream=stream, copy_stream=self.copy_stream)
        if inner:
            inner[2].record(stream)
        self.layer.forward_routed(x, self.idx_t, self.w_t, self.out)
        if inner:
            inner[3].record(stream)
        if record:
            self.paging["hits"] += hits
            self.paging["misses"] += misses
            self.paging["bytes"] += nbytes
            self.paging["copy_ms"] += self.arena.copy_ms()
            self.paging["steps"] += 1

    def close(self):
        if self.paged:
            self.arena.close()
        self.layer.close()


def measure(wl, steps, warmup, world, clocks, peaks, flush_l2, seed, config_name):
    """Warm-up, timed steps, a serialised kernel pass and an end-to-end pass
    of one workload; returns the record (rank-local values are reduced with
    max over ranks)."""
    import torch

    from quantized_routed_expert_04_b200 import binding
    cfg, T, layer = wl.cfg, wl.T, wl.layer
    stream = torch.cuda.current_stream()
    E, S = cfg.n_experts, cfg.n_shared
    for i in range(warmup):
        flush_l2(i)
        wl.step(i)
    torch.cuda.synchronize()
    st, bits = layer.status()
    if int(st) != 0:
        raise RuntimeError("device status %s bits %d" % (st, bits))

    # --- timed region: the forward exactly as a user runs it (consecutive
    # kernels overlap through programmatic dependent launch)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    inner = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    c0 = clocks.mark()
    t_wall = time.perf_counter()
    for i in range(steps):
        flush_l2(i)
        ev[i][0].record(stream)
        wl.step(warmup + i, inner[i] if wl.paged else None, record=True)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    c1 = clocks.mark()
    if world > 1:
        torch.distributed.barrier()
    if wl.paged:  # layer kernels only: routing + forward, not the copies between them
        step_ms = [e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in inner]
    else:
        step_ms = [a.elapsed_time(bb) for a, bb in ev]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), world, "cuda")

    # --- kernel pass: the same steps again with an event pair around every
    # kernel (which serialises them), for per-kernel times and rooflines
    kp_steps = min(steps, 20)
    binding.strata_moe_profile(layer.h, True)
    binding.strata_moe_profile_read(layer.h)
    for i in range(kp_steps):
        flush_l2(i)
        wl.step(warmup + i)
    torch.cuda.synchronize()
    prof = binding.strata_moe_profile_read(layer.h)
    binding.strata_moe_profile(layer.h, False)

    timed_ids = [(warmup + i) % wl.n_batches for i in range(steps)]
    kp_ids = timed_ids[:kp_steps]
    H, I = cfg.hidden, cfg.inter
    B_e = synth.expert_bytes(H, I)
    rec = {"config": config_name, "tokens": T, "steps": steps, "warmup": warmup,
           "ms_per_step": ms, "value": whole_job_tokens_per_s(T, world, ms), "unit": UNIT,
           "wall_s_timed_region": t_wall,
           "phase_ms_per_launch": {k: round(v[1] / max(1, v[0]), 5) for k, v in prof.items()
                                   if v[0]},
           "launches_per_step": sum(v[0] for v in prof.values()) / max(1, kp_steps)}
    rooflines = {}
    if T <= SMALL_T:
        # HBM-bound: algorithmic bytes = the blobs of the distinct routed
        # experts of the batch plus the shared ones, read once
        per = {"gate_up": 2 * I * H * 9 // 16, "down": H * I * 9 // 16, "fused": B_e}
        step_bytes = sum((wl.distinct[j] + S) * B_e for j in timed_ids) / len(timed_ids)
        rec["expert_weight_bytes_per_step"] = step_bytes
        rec["expert_weight_gbs"] = step_bytes / (ms / 1000.0) / 1e9
        rec["expert_weight_frac_of_hbm"] = rec["expert_weight_gbs"] / peaks["hbm"]
        rec["expert_weight_frac_of_8tbs"] = rec["expert_weight_gbs"] / NOMINAL_HBM_GBS
        for ph, unit_bytes in per.items():
            n, tot = prof.get(ph, (0, 0.0))
            if not n:
                continue
            alg = sum((wl.distinct[j] + S) * unit_bytes for j in kp_ids) / len(kp_ids)
            avg = tot / n
            rooflines[ph] = {"bound": "hbm", "achieved": alg / (avg / 1000.0) / 1e9,
                             "peak": peaks["hbm"], "unit": "GB/s",
                             "peak_source": peaks["source"] + " (copy kernel)",
                             "algorithmic_bytes_per_launch": alg, "avg_launch_ms": avg}
        traffic_key, kfiles, traffic_kernel = "decode_fused_%s_t%d" % (config_name, T), \
            KERNEL_SOURCES["decode"], "fused"
    else:
        flops_pair = 6.0 * H * I
        P = T * (cfg.top_k + S)
        rec["tflops"] = flops_pair * P / (ms / 1000.0) / 1e12
        for ph, f in (("gate_up", 4.0 * H * I * P), ("down", 2.0 * H * I * P)):
            n, tot = prof.get(ph, (0, 0.0))
            if not n:
                continue
            avg = tot / n
            ach = f / (avg / 1000.0) / 1e12
            rooflines[ph] = {"bound": "tensor", "achieved": ach, "peak": peaks["tc"],
                             "unit": "TFLOP/s", "peak_source": peaks["source"] +
                             " (dense bf16 GEMM burst; f16 has the same rate)",
                             "frac_of_sustained": ach / peaks["tc_sustained"],
                             "algorithmic_flops_per_launch": f, "avg_launch_ms": avg}
        gu, dn = prof.get("gate_up", (0, 0.0)), prof.get("down", (0, 0.0))
        if gu[0]:
            rec["expert_gemm_tflops"] = flops_pair * P / ((gu[1] + dn[1]) / gu[0] / 1000.0) / 1e12
        traffic_key, kfiles, traffic_kernel = "expert_tc_gateup_%s_t%d" % (config_name, T), \
            KERNEL_SOURCES["prefill"], "gate_up"
    for r in rooflines.values():
        r["frac"] = r["achieved"] / r["peak"]
        r["timing"] = ("CUDA events around every launch, in a pass of %d of the timed steps run "
                       "again right after the timed region (launches serialised)" % kp_steps)
    if rooflines:
        dom = max(rooflines, key=lambda k: rooflines[k]["avg_launch_ms"])
        roof = dict(rooflines[dom], kernel=dom)
        roof["traffic"] = (traffic_from_profile(kfiles, traffic_key) if dom == traffic_kernel
                           else None)
        rec["roofline"] = roof
        rec["rooflines"] = rooflines

    # --- end to end through the C interface with host buffers
    x_host = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    for j, xh in enumerate(x_host):
        xh.copy_(wl.xs[j % wl.n_batches].cpu())
    out_host = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty_like(wl.xs[0])
    e2e_steps = max(10, min(steps, 100))
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        flush_l2(i)
        e2e_ev[i][0].record(stream)
        x_stage.copy_(x_host[i % 4], non_blocking=True)
        wl.step(i, x=x_stage)   # paged: includes the host routing read and the copies
        out_host.copy_(wl.out, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(a.elapsed_time(bb) for a, bb in e2e_ev) / e2e_steps, world,
                            "cuda")
    rec["e2e"] = {"value": whole_job_tokens_per_s(T, world, e2e_ms), "unit": UNIT,
                  "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
                  "ms_per_step": e2e_ms}
    rec["clocks"] = clocks.window(c0, c1)
    st, bits = layer.status()
    if int(st) != 0:
        raise RuntimeError("device status %s bits %d after measurement" % (st, bits))
    if wl.paged:
        n = max(1, wl.paging["steps"])
        rec["paging"] = {
            "n_slots": cfg.n_slots, "note": "layer time (value) excludes the expert copies; "
            "e2e includes them and the host read of the routing",
            "hits_per_step": wl.paging["hits"] / n, "misses_per_step": wl.paging["misses"] / n,
            "copy_bytes_per_step": wl.paging["bytes"] / n,
            "copy_ms_per_step": wl.paging["copy_ms"] / n,
            "copy_gbs": wl.paging["bytes"] / max(wl.paging["copy_ms"], 1e-9) / 1e6}
    return rec


CHUNKS = (1024, 2048, 4096)


def measure_chunked(cfg, T, seed, steps, flush_l2, clocks):
    """Chunked prefill through an arena with half the experts' slots
    (strata_arena_prefill): per chunk size, the device time of whole prompts
    (routing, the host read of the routing, per-chunk expert copies from
    pinned host memory, expert passes and combines), copied bytes and groups."""
    import torch

    from quantized_routed_expert_04_b200 import binding
    E, S = cfg.n_experts, cfg.n_shared
    blobs = synth.make_all_blobs(cfg, seed)
    W, b = synth.make_router(cfg, seed)
    W_dev, b_dev = torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda()
    shared = torch.from_numpy(blobs[E:]).cuda()
    pool = torch.from_numpy(np.ascontiguousarray(blobs[:E]).reshape(-1)).pin_memory()
    B_e = synth.expert_bytes(cfg.hidden, cfg.inter)
    arena_mem = torch.empty(cfg.n_slots * B_e, dtype=torch.uint8, device="cuda")
    x = torch.from_numpy(synth.make_x(cfg, T, seed).view(np.int16)).cuda().view(torch.bfloat16)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    recs = []
    for chunk in CHUNKS:
        layer = binding.StrataMoE(cfg.hidden, cfg.inter, E, cfg.top_k, S, cfg.n_slots)
        layer.set_router(W_dev, b_dev)
        for i in range(S):
            layer.bind_shared(i, shared[i])
        layer.reserve(T)
        arena = binding.Arena(layer, pool, arena_mem)
        arena.prefill(x, chunk, out, copy_stream=copy_stream)      # warm-up
        torch.cuda.synchronize()
        tot = {"ms": 0.0, "bytes": 0, "misses": 0, "hits": 0, "passes": 0, "chunks": 0}
        c0 = clocks.mark()
        for i in range(steps):
            flush_l2(i)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            st = arena.prefill(x, chunk, out, copy_stream=copy_stream)
            e1.record(stream)
            torch.cuda.synchronize()
            tot["ms"] += e0.elapsed_time(e1)
            for key in ("bytes", "misses", "hits", "passes", "chunks"):
                tot[key] += st[key]
        st, bits = layer.status()
        if int(st) != 0:
            raise RuntimeError("chunked prefill status %s bits %d" % (st, bits))
        ms = tot["ms"] / steps
        recs.append({"chunk_tokens": chunk, "tokens": T, "n_slots": cfg.n_slots,
                     "ms_per_step": ms, "value": T / (ms / 1000.0), "unit": UNIT,
                     "copy_bytes_per_step": tot["bytes"] / steps,
                     "expert_copies_per_step": tot["misses"] / steps,
                     "resident_hits_per_step": tot["hits"] / steps,
                     "expert_groups_per_step": tot["passes"] / steps,
                     "chunks_per_step": tot["chunks"] / steps,
                     "clocks": clocks.window(c0, clocks.mark())})
        arena.close()
        layer.close()
    return {"workload": cfg.description, "note": "device time of a whole prompt per chunk size, "
            "copies included (the arena starts each timed prompt with what the previous one "
            "left)", "records": recs}


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        reference_arm(args)
        return
    import datetime

    import torch
    import torch.distributed as dist

    from quantized_routed_expert_04_b200 import binding, build
    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    build.build()
    binding.load_library()
    peaks = load_peaks()

    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    clean = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    sink = torch.empty(1, dtype=torch.float32, device="cuda")

    def flush_l2(i):
        # write a buffer larger than L2, then read another one so that the
        # flush's dirty lines are written back here, outside the timed region
        flush.fill_(float(i))
        torch.sum(clean, dim=0, out=sink.view(()))

    cfg = synth.CONFIGS[args.config]
    T = args.tokens
    with ClockSampler(local) as clocks:
        wl = Workload(cfg, T, args.seed, rank, min(args.warmup + args.steps, 64 if T <= 64 else 8))
        head = measure(wl, args.steps, args.warmup, world, clocks, peaks, flush_l2, args.seed,
                       args.config)
        cpu = None
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cpu = run_cpu_baseline(cfg, wl.blobs, wl.W, wl.b, T, args.seed, corr=wl.corr)
        wl.close()
        del wl
        torch.cuda.empty_cache()
        subs, chunked = [], None
        if args.subrecords:
            for name, t in SUBRECORDS:
                c = synth.CONFIGS[name]
                w = Workload(c, t, args.seed, rank, 64)
                r = measure(w, args.sub_steps, max(args.warmup, 10), world, clocks, peaks,
                            flush_l2, args.seed, name)
                r["config"] = config_desc(c, t, world)
                subs.append(r)
                w.close()
                del w
                torch.cuda.empty_cache()
            chunked = measure_chunked(synth.CONFIGS["prefill_paged"], HEADLINE[1], args.seed,
                                      3, flush_l2, clocks)
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4 weights x f16 activations, f32 accumulate (router f64)",
            "data": "synthetic (seeded, resident in HBM)",
            "config": config_desc(cfg, T, world),
        }
        for k in ("tflops", "expert_gemm_tflops", "expert_weight_gbs", "expert_weight_frac_of_hbm",
                  "expert_weight_frac_of_8tbs", "roofline", "rooflines", "phase_ms_per_launch",
                  "e2e", "paging"):
            if k in head:
                line[k] = head[k]
        line["gpu_launches"] = int(round(head["launches_per_step"] * args.steps))
        line["clocks"] = head["clocks"]
        line["wall_s_timed_region"] = head["wall_s_timed_region"]
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if wl_paged(cfg):
            line["data"] = "synthetic (seeded); %d of %d experts resident, the rest in pinned " \
                           "host memory" % (cfg.n_slots, cfg.n_experts)
        if subs:
            line["decode"] = subs
            line["chunked_prefill"] = chunked
            s0 = clocks.mark()
            line["clocks_whole_run"] = clocks.window(0, s0)
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


def wl_paged(cfg):
    return cfg.n_slots < cfg.n_experts


if __name__ == "__main__":
    main()
