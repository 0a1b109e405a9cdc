"""Chunked prefill through an arena with fewer slots than experts
(strata_arena_prefill), through the C interface: for several chunk sizes --
one chunk, ragged chunks, chunks smaller than a decode batch -- the output is
bit-identical to the all-resident forward of the same tokens (the paged-vs-
resident rule of "How these numbers are measured", "Fidelity"), every chunk
runs one group of experts per arena-full of its distinct experts, and the
copied bytes are whole blobs."""
import numpy as np
import pytest

from quantized_routed_expert_04_b200 import synth
from tests.harness import GpuLayer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_routed_expert_04_b200 import build
    build.build()


def chunk_config(T, n_slots=16):
    # the prefill layer's routing structure at a small size, with an arena of
    # a quarter of the experts
    return synth.custom_config("prefill_arena", 512, 256, 64, 8, n_shared=1, n_slots=n_slots,
                               tokens=(T,), bias="zipf", zipf_s=0.8, zipf_beta=1.0)


@pytest.mark.parametrize("T,chunk", [(2048, 2048), (2048, 1000), (2048, 256), (300, 64)])
def test_chunked_prefill_bitwise_equals_resident(T, chunk):
    import oracle
    import torch

    from quantized_routed_expert_04_b200 import binding
    cfg = chunk_config(T)
    full = GpuLayer(synth.custom_config("prefill_arena", 512, 256, 64, 8, n_shared=1,
                                        tokens=(T,), bias="zipf", zipf_s=0.8, zipf_beta=1.0))
    x = synth.make_x(cfg, T, step=41)
    st, ref = full.forward(x)
    assert int(st[0]) == 0

    E, S = cfg.n_experts, cfg.n_shared
    blobs = full.blobs
    layer = binding.StrataMoE(cfg.hidden, cfg.inter, E, cfg.top_k, S, cfg.n_slots)
    layer.set_router(full.W_dev, full.b_dev)
    for i in range(S):
        layer.bind_shared(i, full.blob_ptr(E + i))
    pool = torch.from_numpy(np.ascontiguousarray(blobs[:E]).reshape(-1)).pin_memory()
    B_e = synth.expert_bytes(cfg.hidden, cfg.inter)
    arena_mem = torch.empty(cfg.n_slots * B_e, dtype=torch.uint8, device="cuda")
    arena = binding.Arena(layer, pool, arena_mem)
    copy_stream = torch.cuda.Stream()
    xd = full.x_dev(x)
    for rep in range(2):   # the second call starts from the arena the first left
        out = torch.zeros_like(xd)
        stats = arena.prefill(xd, chunk, out, copy_stream=copy_stream)
        st, bits = layer.status()
        assert int(st) == 0, (st, bits)
        got = out.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, ref), "chunk %d, call %d" % (chunk, rep)
        _, idx, _ = oracle.route(x, full.W, full.b, cfg.top_k)
        n_chunks = (T + chunk - 1) // chunk
        groups = sum(-(-len(set(idx[c:c + chunk].reshape(-1).tolist())) // cfg.n_slots)
                     for c in range(0, T, chunk))
        assert stats["chunks"] == n_chunks and stats["passes"] == groups, stats
        assert stats["bytes"] == stats["misses"] * B_e
    arena.close()
    layer.close()
    full.close()
