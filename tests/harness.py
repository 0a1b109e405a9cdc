"""Test-side helpers: put a synthetic layer on the GPU through the C interface
and compute the oracle's answer for the same seeded inputs."""
from __future__ import annotations

import numpy as np

from quantized_routed_expert_04_b200 import synth

# Tolerance of the layer output (errors computed in fp32/fp64):
#   max |out - ref| <= 2e-2 * max |ref|  and  sum |out - ref| / sum |ref| <= 2e-3
TOL_MAX = 2e-2
TOL_MEAN = 2e-3


def layer_errors(out_bf16_bits: np.ndarray, ref: np.ndarray):
    out = synth.bf16_bits_to_f32(out_bf16_bits).astype(np.float64)
    ref = ref.astype(np.float64)
    err = np.abs(out - ref)
    return err.max() / max(np.abs(ref).max(), 1e-30), err.sum() / max(np.abs(ref).sum(), 1e-30)


def assert_within_tolerance(out_bf16_bits, ref, what=""):
    mx, mean = layer_errors(out_bf16_bits, ref)
    assert mx <= TOL_MAX and mean <= TOL_MEAN, "%s max-rel %.3e mean-rel %.3e" % (what, mx, mean)
    return mx, mean


class GpuLayer:
    """A layer handle with all blobs resident on the device."""

    def __init__(self, cfg, seed=0, blobs=None, bind="all", perm_index=0, fmt="int4"):
        import torch

        from quantized_routed_expert_04_b200 import binding
        self.torch = torch
        self.cfg = cfg
        self.seed = seed
        self.fmt = fmt
        if blobs is None:
            blobs = synth.make_all_blobs(cfg, seed) if fmt == "int4" else \
                synth.make_all_blobs_nvfp4(cfg, seed)
        self.blobs = blobs
        self.dev_blobs = torch.from_numpy(self.blobs).cuda()
        W, b = synth.make_router(cfg, seed)
        self.W, self.b = W, b
        self.W_dev = torch.from_numpy(W).cuda()
        self.b_dev = None if b is None else torch.from_numpy(b).cuda()
        self.layer = binding.StrataMoE(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k,
                                       cfg.n_shared, cfg.n_slots)
        self.layer.set_router(self.W_dev, self.b_dev)
        if fmt != "int4":
            self.layer.set_format(binding.FORMAT_NVFP4)
        for i in range(cfg.n_shared):
            self.layer.bind_shared(i, self.blob_ptr(cfg.n_experts + i))
        self.slot_expert = np.full(cfg.n_slots, -1, np.int32)
        if bind == "all":
            assert cfg.n_slots == cfg.n_experts
            self.bind_permutation(synth.make_slot_permutation(cfg, seed, perm_index))

    def blob_ptr(self, e):
        return self.dev_blobs[e].data_ptr()

    def bind_permutation(self, perm):
        for s in range(self.cfg.n_slots):
            self.layer.bind_slot(s, -1, None)
        for s, e in enumerate(perm):
            self.layer.bind_slot(s, int(e), self.blob_ptr(int(e)))
        self.slot_expert = np.asarray(perm, np.int32).copy()

    def bind_only(self, experts, rng_seed=0):
        """Empty every slot, then bind just `experts` into random slots."""
        experts = sorted(set(int(e) for e in experts))
        assert len(experts) <= self.cfg.n_slots
        for s in range(self.cfg.n_slots):
            self.layer.bind_slot(s, -1, None)
        slots = np.random.default_rng(rng_seed).permutation(self.cfg.n_slots)[:len(experts)]
        self.slot_expert[:] = -1
        for s, e in zip(slots, experts):
            self.layer.bind_slot(int(s), e, self.blob_ptr(e))
            self.slot_expert[s] = e

    def x_dev(self, x_bits):
        return self.torch.from_numpy(x_bits.view(np.int16)).cuda().view(self.torch.bfloat16)

    def forward(self, x_bits):
        torch = self.torch
        x = self.x_dev(x_bits)
        out = torch.empty_like(x)
        self.layer.forward(x, out)
        st = self.layer.status()
        return st, out.view(torch.int16).cpu().numpy().view(np.uint16)

    def route(self, x_bits):
        torch = self.torch
        T = x_bits.shape[0]
        x = self.x_dev(x_bits)
        logits = torch.empty(T, self.cfg.n_experts, dtype=torch.float32, device="cuda")
        idx = torch.empty(T, self.cfg.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, self.cfg.top_k, dtype=torch.float32, device="cuda")
        self.layer.route(x, logits, idx, w)
        torch.cuda.synchronize()
        return logits.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy()

    def forward_routed(self, x_bits, idx, w):
        torch = self.torch
        x = self.x_dev(x_bits)
        out = torch.empty_like(x)
        self.layer.forward_routed(x, torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda(),
                                  torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda(), out)
        st = self.layer.status()
        return st, out.view(torch.int16).cpu().numpy().view(np.uint16)

    def close(self):
        self.layer.close()


def oracle_reference_parallel(cfg, blobs, W, b, x_bits, idx=None, w=None, n_threads=None,
                              fmt="int4"):
    """oracle_reference split over token chunks run in threads (the oracle's
    C calls release the interpreter lock, so the chunks run in parallel on
    the host cores).  Each token's output depends only on that token, so the
    result equals the single call's.  Returns (out, idx, w)."""
    import concurrent.futures
    import os

    import oracle
    T = x_bits.shape[0]
    if idx is None:
        _, idx, w = oracle.route(x_bits, W, b, cfg.top_k)
    n = max(1, min(T, n_threads or os.cpu_count() or 1))
    bounds = np.linspace(0, T, n + 1).astype(int)
    out = np.zeros((T, cfg.hidden), np.float32)

    def run(i):
        lo, hi = bounds[i], bounds[i + 1]
        if hi > lo:
            out[lo:hi] = oracle_reference(cfg, blobs, W, b, x_bits[lo:hi], idx[lo:hi],
                                          w[lo:hi], fmt=fmt)[0]

    with concurrent.futures.ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(run, range(n)))
    return out, idx, w


def oracle_reference(cfg, blobs, W, b, x_bits, idx=None, w=None, fmt="int4"):
    """Oracle output (fp32 [T][H]) with every expert bound; routing computed
    by the oracle unless idx/w are given.  Returns (out, idx, w)."""
    import oracle
    E, S = cfg.n_experts, cfg.n_shared
    se = np.arange(E, dtype=np.int32)
    sb = [blobs[e] for e in range(E)]
    shared = [blobs[E + i] for i in range(S)]
    if idx is None:
        _, idx, w = oracle.route(x_bits, W, b, cfg.top_k)
    st, out = oracle.forward_routed(x_bits, cfg.hidden, cfg.inter, E, cfg.top_k, se, sb, shared,
                                    idx, w, fmt=fmt)
    assert st == oracle.OK
    return out, idx, w
