"""Expert arena (LRU residency over the slot table) on the GPU.

Checks, step by step over a stream of decode batches, that
  * the arena's hits, misses and slot choices equal an independent model of
    the stated policy (lowest empty slot, else least recently used slot not
    asked for now, ties to the lowest slot);
  * the layer's output through the arena is bit-identical to the output of a
    layer with every expert resident (the paged-vs-resident fidelity rule of
    "How these numbers are measured");
  * requests the arena cannot serve are refused without side effects."""
import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth

pytestmark = pytest.mark.gpu


class LruModel:
    def __init__(self, n_slots):
        self.n = n_slots
        self.slot_of = {}
        self.expert_in = [-1] * n_slots
        self.last = [0] * n_slots
        self.tick = 0

    def ensure(self, ids):
        distinct = list(dict.fromkeys(int(e) for e in ids))
        assert len(distinct) <= self.n
        self.tick += 1
        hits = misses = 0
        for e in distinct:
            if e in self.slot_of:
                self.last[self.slot_of[e]] = self.tick
                hits += 1
        for e in distinct:
            if e in self.slot_of:
                continue
            empty = [s for s in range(self.n) if self.expert_in[s] < 0]
            if empty:
                victim = empty[0]
            else:
                victim = min((s for s in range(self.n) if self.last[s] != self.tick),
                             key=lambda s: (self.last[s], s))
            old = self.expert_in[victim]
            if old >= 0:
                del self.slot_of[old]
            self.expert_in[victim] = e
            self.slot_of[e] = victim
            self.last[victim] = self.tick
            misses += 1
        return hits, misses


def _cfg():
    # the wide-expert decode layer's structure at a small size: many experts,
    # a Zipf-skewed router and an arena of a quarter of them
    return synth.custom_config("arena", 1024, 512, 64, 6, n_shared=0, n_slots=16, tokens=(2,),
                               bias="zipf", zipf_s=1.1, zipf_beta=synth.WIDE_ZIPF_BETA)


def test_arena_lru_policy_and_fidelity():
    import torch

    from quantized_routed_expert_04_b200 import binding
    cfg = _cfg()
    E, T, k = cfg.n_experts, 2, cfg.top_k
    blobs = synth.make_all_blobs(cfg, seed=3)
    B = blobs.shape[1]
    W, b = synth.make_router(cfg, seed=3)
    W_dev, b_dev = torch.from_numpy(W).cuda(), torch.from_numpy(b).cuda()

    # reference: every expert resident
    ref = binding.StrataMoE(cfg.hidden, cfg.inter, E, k, 0, E)
    ref.set_router(W_dev, b_dev)
    dev_all = torch.from_numpy(blobs).cuda()
    for e in range(E):
        ref.bind_slot(e, e, dev_all[e])

    # paged: 16 slots filled from a pinned host pool
    lay = binding.StrataMoE(cfg.hidden, cfg.inter, E, k, 0, cfg.n_slots)
    lay.set_router(W_dev, b_dev)
    pool = torch.from_numpy(blobs.reshape(-1)).pin_memory()
    arena_mem = torch.empty(cfg.n_slots * B, dtype=torch.uint8, device="cuda")
    arena = binding.Arena(lay, pool, arena_mem)
    model = LruModel(cfg.n_slots)
    copy_stream = torch.cuda.Stream()
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    total_misses = 0
    for step in range(12):
        x = torch.from_numpy(synth.make_x(cfg, T, seed=3, step=step).view(np.int16)).cuda() \
            .view(torch.bfloat16)
        lay.route(x, None, idx, w)
        ids = idx.cpu().numpy().reshape(-1)
        hits, misses, nbytes = arena.ensure(ids, copy_stream=copy_stream)
        assert (hits, misses) == model.ensure(ids), step
        assert nbytes == misses * B
        total_misses += misses
        for e in range(E):
            assert arena.slot_of(e) == model.slot_of.get(e, -1), (step, e)
        out = torch.empty_like(x)
        lay.forward_routed(x, idx, w, out)
        assert int(lay.status()[0]) == 0
        out_ref = torch.empty_like(x)
        ref.forward(x, out_ref)
        assert int(ref.status()[0]) == 0
        assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16)), step
        assert arena.copy_ms() >= 0.0
    assert total_misses > cfg.n_slots  # evictions happened

    # refusals change nothing
    before = [arena.slot_of(e) for e in range(E)]
    with pytest.raises(binding.StrataError) as err:
        arena.ensure(list(range(cfg.n_slots + 1)))
    assert err.value.status == binding.Status.TOO_MANY_EXPERTS
    with pytest.raises(binding.StrataError) as err:
        arena.ensure([0, E])
    assert err.value.status == binding.Status.INVALID_ARG
    assert [arena.slot_of(e) for e in range(E)] == before
    arena.close()
    lay.close()
    ref.close()
